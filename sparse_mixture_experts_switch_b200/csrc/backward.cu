// Backward pass of the top-1 Switch-FFN layer, the parts around the expert
// GEMMs ("Switch Transformers: scaling to trillion-parameter models"):
//   * the gate-scaled gather of the output gradient into the capacity
//     buffers (section "Switch Routing: From Top-k to k = 1", combine
//     equation: out = x + p_idx E_idx(x), so dE = p_idx dout);
//   * the router backward: the gate gradient dout . E(x) reaches the logits
//     through the softmax (the gate equation), together with the gradient of
//     the load-balancing loss through P_i (section "The Load-Balancing
//     Loss"; f_i is piecewise constant);
//   * the input gradient of dropped tokens (residual and router only).
// Router arithmetic is fp32 on CUDA cores (no TF32), every reduction in a
// fixed order.
#include "backward.cuh"

namespace smoe {

namespace {

constexpr int kWarpsPerBlock = 8;

__device__ __forceinline__ uint32_t scale_bf16x2(uint32_t w, float g) {
  return pack_bf16x2(bf16_lo(w) * g, bf16_hi(w) * g);
}

// One warp per slot row.
__global__ void __launch_bounds__(256) bwd_gather_kernel(int64_t S, int64_t C, int d, int F,
                                                         const int* __restrict__ counts,
                                                         const int* __restrict__ slot_token,
                                                         const float* __restrict__ gate,
                                                         const uint4* __restrict__ dout,
                                                         uint4* __restrict__ dys,
                                                         uint4* __restrict__ hbuf) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t s = static_cast<int64_t>(blockIdx.x) * kWarpsPerBlock + warp;
  if (s >= S) return;
  const int64_t e = s / C;
  const int64_t r = s - e * C;
  const int64_t cnt = counts[e];
  const int64_t ne = cnt < C ? cnt : C;
  const int dv = d / 8;
  uint4* drow = dys + s * dv;
  if (r < ne) {
    const int64_t t = slot_token[s];
    const float g = gate[t];
    const uint4* src = dout + t * dv;
    for (int v = lane; v < dv; v += 32) {
      const uint4 u = __ldg(src + v);
      drow[v] = make_uint4(scale_bf16x2(u.x, g), scale_bf16x2(u.y, g), scale_bf16x2(u.z, g),
                           scale_bf16x2(u.w, g));
    }
    return;
  }
  for (int v = lane; v < dv; v += 32) drow[v] = make_uint4(0, 0, 0, 0);
  const int64_t up = (ne + 63) / 64 * 64;
  if (r < (up < C ? up : C)) {
    const int fv = F / 8;
    uint4* hrow = hbuf + s * fv;
    for (int v = lane; v < fv; v += 32) hrow[v] = make_uint4(0, 0, 0, 0);
  }
}

// One warp per token.
__global__ void __launch_bounds__(256) router_bwd_dh_kernel(
    int64_t T, int N, int64_t C, int ntn, const float* __restrict__ probs,
    const int* __restrict__ idx, const int* __restrict__ rank, const uint8_t* __restrict__ drop,
    const float* __restrict__ gate, const float* __restrict__ dgp, const int* __restrict__ counts,
    float loss_scale, float* __restrict__ dh, float* __restrict__ dgate) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kWarpsPerBlock + warp;
  if (t >= T) return;
  const bool kept = drop[t] == 0;
  const int e = idx[t];
  float dg = 0.f;
  if (kept) {
    const int64_t s = static_cast<int64_t>(e) * C + rank[t];
    float sum = 0.f;
    for (int j = 0; j < ntn; ++j) sum += dgp[s * ntn + j];     // fixed order
    dg = sum / gate[t];
  }
  const float* prow = probs + t * N;
  float acc = 0.f;
  for (int i = lane; i < N; i += 32) {
    const float dp = loss_scale * static_cast<float>(counts[i]) + ((kept && i == e) ? dg : 0.f);
    acc = fmaf(prow[i], dp, acc);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  float* hrow = dh + t * N;
  for (int i = lane; i < N; i += 32) {
    const float dp = loss_scale * static_cast<float>(counts[i]) + ((kept && i == e) ? dg : 0.f);
    hrow[i] = prow[i] * (dp - acc);
  }
  if (dgate != nullptr && lane == 0) dgate[t] = dg;
}

constexpr int kSB = 64, kSK = 16;

// dxr [T, d] = dh [T, N] . W_r [N, d]; grid (ceil(T/64), ceil(d/64)),
// 256 threads, 4 x 4 outputs each.
__global__ void __launch_bounds__(256) router_bwd_dx_kernel(int64_t T, int N, int d,
                                                            const float* __restrict__ dh,
                                                            const float* __restrict__ wr,
                                                            float* __restrict__ dxr) {
  __shared__ float As[kSK][kSB + 4];
  __shared__ float Bs[kSK][kSB + 4];
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kSB;
  const int k0 = blockIdx.y * kSB;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int i0 = 0; i0 < N; i0 += kSK) {
    for (int q = threadIdx.x; q < kSB * kSK; q += 256) {
      const int rr = q / kSK, kk = q % kSK;
      As[kk][rr] = (t0 + rr < T && i0 + kk < N) ? dh[(t0 + rr) * N + i0 + kk] : 0.f;
      const int kb = q / kSB, cc = q % kSB;
      Bs[kb][cc] = (i0 + kb < N && k0 + cc < d) ? wr[static_cast<int64_t>(i0 + kb) * d + k0 + cc]
                                                : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kSK; ++kk) {
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
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t t = t0 + ty * 4 + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int k = k0 + tx * 4 + j;
      if (k < d) dxr[t * d + k] = acc[i][j];
    }
  }
}

constexpr int64_t kDwChunk = 2048;     // tokens per split-K chunk

int64_t dw_chunks(int64_t T) { return (T + kDwChunk - 1) / kDwChunk; }

// part[c][i][k] = sum over tokens t of chunk c of dh[t, i] x[t, k];
// partb[c][i] = sum over the chunk of dh[t, i].  grid (ceil(N/64),
// ceil(d/64), chunks).
__global__ void __launch_bounds__(256) router_bwd_dw_kernel(int64_t T, int N, int d,
                                                            const float* __restrict__ dh,
                                                            const __nv_bfloat16* __restrict__ x,
                                                            float* __restrict__ part,
                                                            float* __restrict__ partb) {
  __shared__ float As[kSK][kSB + 4];
  __shared__ float Bs[kSK][kSB + 4];
  const int i0 = blockIdx.x * kSB;
  const int k0 = blockIdx.y * kSB;
  const int64_t c = blockIdx.z;
  const int64_t tb = c * kDwChunk;
  const int64_t te = tb + kDwChunk < T ? tb + kDwChunk : T;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  float sb = 0.f;
  for (int64_t u0 = tb; u0 < te; u0 += kSK) {
    for (int q = threadIdx.x; q < kSB * kSK; q += 256) {
      const int kk = q / kSB, cc = q % kSB;
      const int64_t t = u0 + kk;
      As[kk][cc] = (t < te && i0 + cc < N) ? dh[t * N + i0 + cc] : 0.f;
      Bs[kk][cc] = (t < te && k0 + cc < d) ? __bfloat162float(x[t * d + k0 + cc]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kSK; ++kk) {
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
    if (blockIdx.y == 0 && threadIdx.x < kSB) {
#pragma unroll
      for (int kk = 0; kk < kSK; ++kk) sb += As[kk][threadIdx.x];
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int ii = i0 + ty * 4 + i;
    if (ii >= N) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int k = k0 + tx * 4 + j;
      if (k < d) part[(c * N + ii) * d + k] = acc[i][j];
    }
  }
  if (blockIdx.y == 0 && threadIdx.x < kSB && i0 + static_cast<int>(threadIdx.x) < N)
    partb[c * N + i0 + threadIdx.x] = sb;
}

// dw_r[i, k] = sum_c part[c][i][k] in chunk order; db[i] likewise.
__global__ void router_bwd_reduce_kernel(int64_t nch, int N, int d, const float* __restrict__ part,
                                         const float* __restrict__ partb, float* __restrict__ dw_r,
                                         float* __restrict__ db) {
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t nd = static_cast<int64_t>(N) * d;
  if (j < nd) {
    float s = 0.f;
    for (int64_t c = 0; c < nch; ++c) s += part[c * nd + j];
    dw_r[j] = s;
  }
  if (db != nullptr && j < N) {
    float s = 0.f;
    for (int64_t c = 0; c < nch; ++c) s += partb[c * N + j];
    db[j] = s;
  }
}

// One warp per token; only dropped tokens are written.
__global__ void __launch_bounds__(256) bwd_dropped_kernel(int64_t T, int d,
                                                          const uint8_t* __restrict__ drop,
                                                          const uint4* __restrict__ dout,
                                                          const float4* __restrict__ dxr,
                                                          uint4* __restrict__ dx, int residual) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kWarpsPerBlock + warp;
  if (t >= T || drop[t] == 0) return;
  const int dv = d / 8;
  for (int v = lane; v < dv; v += 32) {
    const float4 a = dxr[(t * dv + v) * 2];
    const float4 b = dxr[(t * dv + v) * 2 + 1];
    float o[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    if (residual) {
      const uint4 g = dout[t * dv + v];
      o[0] += bf16_lo(g.x); o[1] += bf16_hi(g.x);
      o[2] += bf16_lo(g.y); o[3] += bf16_hi(g.y);
      o[4] += bf16_lo(g.z); o[5] += bf16_hi(g.z);
      o[6] += bf16_lo(g.w); o[7] += bf16_hi(g.w);
    }
    dx[t * dv + v] = make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]),
                                pack_bf16x2(o[4], o[5]), pack_bf16x2(o[6], o[7]));
  }
}

unsigned warp_blocks(int64_t rows) {
  return static_cast<unsigned>((rows + kWarpsPerBlock - 1) / kWarpsPerBlock);
}

}  // namespace

cudaError_t launch_bwd_gather(int64_t C, int N, int d, int F, const int* counts,
                              const int* slot_token, const float* gate, const void* dout,
                              void* dys, void* hbuf, cudaStream_t st) {
  const int64_t S = static_cast<int64_t>(N) * C;
  if (S == 0) return cudaSuccess;
  bwd_gather_kernel<<<warp_blocks(S), 256, 0, st>>>(
      S, C, d, F, counts, slot_token, gate, static_cast<const uint4*>(dout),
      static_cast<uint4*>(dys), static_cast<uint4*>(hbuf));
  return cudaGetLastError();
}

cudaError_t launch_router_bwd_dh(int64_t T, int N, int64_t C, int ntn, const float* probs,
                                 const int* idx, const int* rank, const uint8_t* drop,
                                 const float* gate, const float* dgp, const int* counts,
                                 float loss_scale, float* dh, float* dgate, cudaStream_t st) {
  router_bwd_dh_kernel<<<warp_blocks(T), 256, 0, st>>>(T, N, C, ntn, probs, idx, rank, drop, gate,
                                                       dgp, counts, loss_scale, dh, dgate);
  return cudaGetLastError();
}

cudaError_t launch_router_bwd_dx(int64_t T, int N, int d, const float* dh, const float* w_r,
                                 float* dxr, cudaStream_t st) {
  const dim3 grid(static_cast<unsigned>((T + kSB - 1) / kSB), static_cast<unsigned>((d + kSB - 1) / kSB));
  router_bwd_dx_kernel<<<grid, 256, 0, st>>>(T, N, d, dh, w_r, dxr);
  return cudaGetLastError();
}

size_t router_bwd_part_floats(int64_t T, int N, int d) {
  return static_cast<size_t>(dw_chunks(T)) * static_cast<size_t>(N) * (static_cast<size_t>(d) + 1);
}

cudaError_t launch_router_bwd_dw(int64_t T, int N, int d, const float* dh, const void* x,
                                 float* part, float* dw_r, float* db, cudaStream_t st) {
  const int64_t nch = dw_chunks(T);
  float* partb = part + nch * N * static_cast<int64_t>(d);
  const dim3 grid(static_cast<unsigned>((N + kSB - 1) / kSB), static_cast<unsigned>((d + kSB - 1) / kSB),
                  static_cast<unsigned>(nch));
  router_bwd_dw_kernel<<<grid, 256, 0, st>>>(T, N, d, dh, static_cast<const __nv_bfloat16*>(x),
                                             part, partb);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t nd = static_cast<int64_t>(N) * d;
  router_bwd_reduce_kernel<<<static_cast<unsigned>((nd + 255) / 256), 256, 0, st>>>(
      nch, N, d, part, partb, dw_r, db);
  return cudaGetLastError();
}

cudaError_t launch_bwd_dropped(int64_t T, int d, const uint8_t* drop, const void* dout,
                               const float* dxr, void* dx, bool residual, cudaStream_t st) {
  bwd_dropped_kernel<<<warp_blocks(T), 256, 0, st>>>(
      T, d, drop, static_cast<const uint4*>(dout), reinterpret_cast<const float4*>(dxr),
      static_cast<uint4*>(dx), residual ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace smoe
