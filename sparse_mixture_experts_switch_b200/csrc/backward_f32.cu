// Backward pass of the Switch-FFN layer in fp32 ("Switch Transformers:
// scaling to trillion-parameter models", section "The Core Idea": N
// independent ReLU FFNs over each expert's capacity buffer; section
// "Switch Routing": out = x + sum over the kept routes of p_i E_i(x), so
// dE_i = p_i dout and the gate p_i receives dout . E_i(x)), on CUDA-core FMA
// tiles like the fp32 forward: the configuration the pages run in full
// precision is small, and fp32 operands have no exact tensor-core form.
//
// One batched GEMM kernel, D[e] = A[e] B[e] over an expert batch, with
// strided operands (either may be stored transposed), B rows optionally
// gathered through slot_token, the M rows or the K length of an expert
// taken from its kept-slot count, and two epilogues: a plain store, and the
// dH epilogue (dA = acc where H > 0, plus the slot's partial gate gradient
// over the tile's 64 columns).  Every output element is one thread's
// fixed-order K loop and every partial sum is added in a fixed order, so
// the gradients are bit-reproducible.
#include "backward.cuh"

namespace smoe {

namespace {

constexpr int kFB = 64, kFK = 16;        // 64 x 64 output tile, K in steps of 16

struct F32Gemm {
  int M, N, K;                  // M, N: output extent; K: reduction length
  int ragged_m, ragged_k;       // M (or K) of expert e is min(counts[e], C)
  const int* counts;
  int64_t C;
  const float* a;               // A(m, k) = a[e * a_e + m * a_m + k * a_k]
  int64_t a_e, a_m, a_k;
  const float* b;               // B(k, n) = b[e * b_e + row * b_k + n]
  int64_t b_e, b_k;             //   row = k, or slot_token[e * C + k] when gathered
  const int* b_gather;
  float* out;                   // out[e * o_e + m * o_m + n]
  int64_t o_e, o_m;
  int dh_epi;                   // dH epilogue: out = acc where h > 0, dgp partials
  const float* h;               //   h[e * o_e + m * o_m + n]
  float* dgp;                   //   dgp[(e * C + m) * ntn + blockIdx.y]
  int ntn;
};

__global__ void __launch_bounds__(256) f32_gemm_kernel(F32Gemm g) {
  __shared__ float As[kFK][kFB + 4];
  __shared__ float Bs[kFK][kFB + 4];
  __shared__ float part[kFB][17];
  const int e = blockIdx.z;
  int64_t kept = g.C;
  if (g.ragged_m || g.ragged_k) {
    const int64_t cnt = g.counts[e];
    kept = cnt < g.C ? cnt : g.C;
  }
  const int M = g.ragged_m ? static_cast<int>(kept) : g.M;
  const int K = g.ragged_k ? static_cast<int>(kept) : g.K;
  const int m0 = blockIdx.x * kFB, n0 = blockIdx.y * kFB;
  if (m0 >= M) return;                                   // uniform for the block
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const float* aE = g.a + static_cast<int64_t>(e) * g.a_e;
  const float* bE = g.b + static_cast<int64_t>(e) * g.b_e;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += kFK) {
    for (int i = threadIdx.x; i < kFB * kFK; i += 256) {
      const int rr = i / kFK, kk = i % kFK;              // A: row rr of the tile
      const int m = m0 + rr, k = k0 + kk;
      As[kk][rr] = (m < M && k < K) ? aE[m * g.a_m + k * g.a_k] : 0.f;
      const int kb = i / kFB, nn = i % kFB;              // B: row kb, column nn
      const int kr = k0 + kb, n = n0 + nn;
      float v = 0.f;
      if (kr < K && n < g.N) {
        const int64_t row = g.b_gather ? g.b_gather[static_cast<int64_t>(e) * g.C + kr] : kr;
        v = bE[row * g.b_k + n];
      }
      Bs[kb][nn] = v;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kFK; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
  float* oE = g.out + static_cast<int64_t>(e) * g.o_e;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    float dot = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (m >= M || n >= g.N) continue;
      const int64_t o = static_cast<int64_t>(m) * g.o_m + n;
      if (g.dh_epi) {
        const float hv = g.h[static_cast<int64_t>(e) * g.o_e + o];
        dot = fmaf(acc[i][j], hv, dot);
        oE[o] = hv > 0.f ? acc[i][j] : 0.f;
      } else {
        oE[o] = acc[i][j];
      }
    }
    if (g.dh_epi) part[ty * 4 + i][tx] = dot;
  }
  if (!g.dh_epi) return;
  __syncthreads();
  // the row's 16 column groups added in order
  if (threadIdx.x < kFB) {
    const int m = m0 + threadIdx.x;
    if (m < M) {
      float s = 0.f;
      for (int t = 0; t < 16; ++t) s += part[threadIdx.x][t];
      g.dgp[(static_cast<int64_t>(e) * g.C + m) * g.ntn + blockIdx.y] = s;
    }
  }
}

cudaError_t run_f32_gemm(const F32Gemm& g, int batches, int m_max, cudaStream_t st) {
  if (batches == 0 || m_max == 0 || g.N == 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>((m_max + kFB - 1) / kFB),
                  static_cast<unsigned>((g.N + kFB - 1) / kFB), static_cast<unsigned>(batches));
  f32_gemm_kernel<<<grid, 256, 0, st>>>(g);
  return cudaGetLastError();
}

// dys[s] = g * dout[t] for kept slot s of token t (g the slot's route's
// gate, as the bf16 gather), zero for padding.  One warp per slot.
__global__ void __launch_bounds__(256) gather_f32_kernel(int64_t S, int64_t C, int d,
                                                         const int* __restrict__ counts,
                                                         const int* __restrict__ slot_token,
                                                         const float* __restrict__ gate,
                                                         const int* __restrict__ idx, int64_t T2,
                                                         const float* __restrict__ dout,
                                                         float* __restrict__ dys) {
  const int64_t s = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (s >= S) return;
  const int64_t e = s / C, r = s - e * C;
  const int64_t cnt = counts[e];
  float* row = dys + s * d;
  if (r < (cnt < C ? cnt : C)) {
    const int64_t t = slot_token[s];
    const float g = (T2 > 0 && idx[t] != e) ? gate[T2 + t] : gate[t];
    for (int k = lane; k < d; k += 32) row[k] = g * dout[t * d + k];
  } else {
    for (int k = lane; k < d; k += 32) row[k] = 0.f;
  }
}

// dx[t] = (residual ? dout[t] : 0) + sum over the token's kept routes of
// dxs[slot] (route order) + sum_i dh[t, i] W_r[i] (expert order).  One warp
// per token, lanes over columns.
__global__ void __launch_bounds__(256) dx_f32_kernel(int64_t T, int routes, int N, int d,
                                                     int64_t C, const int* __restrict__ idx,
                                                     const int* __restrict__ rank,
                                                     const uint8_t* __restrict__ drop,
                                                     const float* __restrict__ dxs,
                                                     const float* __restrict__ dh,
                                                     const float* __restrict__ w_r,
                                                     const float* __restrict__ dout,
                                                     float* __restrict__ dx, int residual) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  int64_t slot[2] = {-1, -1};
  for (int r = 0; r < routes; ++r) {
    const int64_t a = r * T + t;
    if (drop[a] == 0) slot[r] = static_cast<int64_t>(idx[a]) * C + rank[a];
  }
  const float* dht = dh + t * N;
  for (int k = lane; k < d; k += 32) {
    float v = residual ? dout[t * d + k] : 0.f;
    for (int r = 0; r < routes; ++r)
      if (slot[r] >= 0) v += dxs[slot[r] * d + k];
    float rt = 0.f;
    for (int i = 0; i < N; ++i) rt = fmaf(dht[i], w_r[static_cast<int64_t>(i) * d + k], rt);
    dx[t * d + k] = v + rt;
  }
}

// db[i] = sum_t dh[t, i]: one warp per expert, lanes over tokens, then a
// fixed butterfly.
__global__ void __launch_bounds__(256) colsum_f32_kernel(int64_t T, int N,
                                                         const float* __restrict__ dh,
                                                         float* __restrict__ db) {
  const int i = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (i >= N) return;
  float s = 0.f;
  for (int64_t t = lane; t < T; t += 32) s += dh[t * N + i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) db[i] = s;
}

}  // namespace

int bwd_f32_dgp_parts(int F) { return (F + kFB - 1) / kFB; }

cudaError_t launch_bwd_f32_experts(const BwdF32Args& a, cudaStream_t st) {
  const int64_t S = static_cast<int64_t>(a.N) * a.C;
  if (S > 0) {
    gather_f32_kernel<<<static_cast<unsigned>((S + 7) / 8), 256, 0, st>>>(
        S, a.C, a.d, a.counts, a.slot_token, a.gate, a.idx, a.T2, a.dout, a.dys);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const int cap = static_cast<int>(a.C);
  // dA = (dY W2_e) where H > 0, and the gate-gradient partials
  F32Gemm g{};
  g.counts = a.counts;
  g.C = a.C;
  g.N = a.F;
  g.K = a.d;
  g.ragged_m = 1;
  g.a = a.dys;  g.a_e = a.C * a.d;  g.a_m = a.d;  g.a_k = 1;
  g.b = a.w2;   g.b_e = static_cast<int64_t>(a.d) * a.F;  g.b_k = a.F;
  g.out = a.da; g.o_e = a.C * a.F;  g.o_m = a.F;
  g.dh_epi = 1;
  g.h = a.h;
  g.dgp = a.dgp;
  g.ntn = bwd_f32_dgp_parts(a.F);
  cudaError_t e = run_f32_gemm(g, a.N, cap, st);
  if (e != cudaSuccess) return e;
  // dW2_e [d, F] = dY_e^T H_e (K = the expert's kept slots)
  F32Gemm w2{};
  w2.counts = a.counts;
  w2.C = a.C;
  w2.M = a.d;
  w2.N = a.F;
  w2.ragged_k = 1;
  w2.a = a.dys;  w2.a_e = a.C * a.d;  w2.a_m = 1;  w2.a_k = a.d;
  w2.b = a.h;    w2.b_e = a.C * a.F;  w2.b_k = a.F;
  w2.out = a.dw2;  w2.o_e = static_cast<int64_t>(a.d) * a.F;  w2.o_m = a.F;
  e = run_f32_gemm(w2, a.N, a.d, st);
  if (e != cudaSuccess) return e;
  // dW1_e [F, d] = dA_e^T X_e (token rows gathered through slot_token)
  F32Gemm w1{};
  w1.counts = a.counts;
  w1.C = a.C;
  w1.M = a.F;
  w1.N = a.d;
  w1.ragged_k = 1;
  w1.a = a.da;  w1.a_e = a.C * a.F;  w1.a_m = 1;  w1.a_k = a.F;
  w1.b = a.x;   w1.b_e = 0;  w1.b_k = a.d;  w1.b_gather = a.slot_token;
  w1.out = a.dw1;  w1.o_e = static_cast<int64_t>(a.F) * a.d;  w1.o_m = a.d;
  e = run_f32_gemm(w1, a.N, a.F, st);
  if (e != cudaSuccess) return e;
  // dX rows per kept slot: dA W1_e
  F32Gemm xs{};
  xs.counts = a.counts;
  xs.C = a.C;
  xs.N = a.d;
  xs.K = a.F;
  xs.ragged_m = 1;
  xs.a = a.da;  xs.a_e = a.C * a.F;  xs.a_m = a.F;  xs.a_k = 1;
  xs.b = a.w1;  xs.b_e = static_cast<int64_t>(a.F) * a.d;  xs.b_k = a.d;
  xs.out = a.dxs;  xs.o_e = a.C * a.d;  xs.o_m = a.d;
  return run_f32_gemm(xs, a.N, cap, st);
}

cudaError_t launch_bwd_f32_router(const BwdF32Args& a, int routes, const int* rank,
                                  const uint8_t* drop, const float* dh, const float* w_r,
                                  float* dw_r, float* db_r, float* dx, bool residual,
                                  cudaStream_t st) {
  // dW_r [N, d] = dh^T x, one batch, K = T
  F32Gemm r{};
  r.M = a.N;
  r.N = a.d;
  r.K = static_cast<int>(a.T);
  r.C = 0;
  r.a = dh;  r.a_e = 0;  r.a_m = 1;  r.a_k = a.N;
  r.b = a.x;  r.b_e = 0;  r.b_k = a.d;
  r.out = dw_r;  r.o_e = 0;  r.o_m = a.d;
  cudaError_t e = run_f32_gemm(r, 1, a.N, st);
  if (e != cudaSuccess) return e;
  if (db_r) {
    colsum_f32_kernel<<<static_cast<unsigned>((a.N + 7) / 8), 256, 0, st>>>(a.T, a.N, dh, db_r);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  dx_f32_kernel<<<static_cast<unsigned>((a.T + 7) / 8), 256, 0, st>>>(
      a.T, routes, a.N, a.d, a.C, a.idx, rank, drop, a.dxs, dh, w_r, a.dout, dx,
      residual ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace smoe
