// Backward pass of the Switch-FFN layer, the parts around the expert GEMMs
// ("Switch Transformers: scaling to trillion-parameter models"):
//   * the gate-scaled gather of the output gradient into the capacity
//     buffers (section "Switch Routing: From Top-k to k = 1", combine
//     equation: out = x + p_idx E_idx(x), so dE = p_idx dout);
//   * the router backward: the gate gradient dout . E(x) reaches the logits
//     through the softmax (the gate equation), together with the gradient of
//     the load-balancing loss through P_i (section "The Load-Balancing
//     Loss"; f_i is piecewise constant);
//   * the input gradient of dropped tokens (residual and router only);
//   * top-2 (section "Switch Routing": out = x + sum over the top-k set of
//     p_i E_i(x), p not renormalised): each kept route has its own gate and
//     gate gradient, and a token's two slots' input gradients are added.
// dh is formed in fp32 and split into hi + lo bf16 planes for the tensor
// cores (the products with bf16 x, or with W_r's own hi + lo split, are then
// exact to about 2^-17 relative); every reduction runs in a fixed order.
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
                                                         const int* __restrict__ idx, int64_t T2,
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
    // top-2: the slot's route is the token's first choice if that is e
    const float g = (T2 > 0 && idx[t] != e) ? gate[T2 + t] : gate[t];
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
    int64_t T, int N, int Np, int64_t C, int64_t S, int ntn, const float* __restrict__ probs,
    const int* __restrict__ idx, const int* __restrict__ rank, const uint8_t* __restrict__ drop,
    const float* __restrict__ gate, const float* __restrict__ dgp, const int* __restrict__ counts,
    float loss_scale, float* __restrict__ dh, __nv_bfloat16* __restrict__ dhp,
    __nv_bfloat16* __restrict__ dhs, float* __restrict__ dgate, int* __restrict__ drop_list,
    int* __restrict__ n_drop) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kWarpsPerBlock + warp;
  if (t >= T) return;
  const bool kept = drop[t] == 0;
  const int e = idx[t];
  const int64_t s = static_cast<int64_t>(e) * C + rank[t];     // the token's slot if kept
  float dg = 0.f;
  if (kept) {
    float sum = 0.f;
    for (int j = 0; j < ntn; ++j) sum += dgp[s * ntn + j];     // fixed order
    dg = sum / gate[t];
  } else if (lane == 0) {
    drop_list[atomicAdd(n_drop, 1)] = static_cast<int>(t);
  }
  const float* prow = probs + t * N;
  float acc = 0.f;
  for (int i = lane; i < N; i += 32) {
    const float dp = loss_scale * static_cast<float>(counts[i]) + ((kept && i == e) ? dg : 0.f);
    acc = fmaf(prow[i], dp, acc);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  __syncwarp();
  for (int i = lane; i < Np; i += 32) {
    float v = 0.f;
    if (i < N) {
      const float dp = loss_scale * static_cast<float>(counts[i]) + ((kept && i == e) ? dg : 0.f);
      v = prow[i] * (dp - acc);
      dh[t * N + i] = v;
    }
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
    dhp[t * Np + i] = hi;
    dhp[T * Np + t * Np + i] = lo;
    if (kept) {
      dhs[s * Np + i] = hi;
      dhs[S * Np + s * Np + i] = lo;
    }
  }
  if (dgate != nullptr && lane == 0) dgate[t] = dg;
}

// One warp per token (top-2): both routes' gate gradients, dp, dh and its
// planes; the router term's planes go to the first kept slot only.
__global__ void __launch_bounds__(256) router_bwd_dh_top2_kernel(
    int64_t T, int N, int Np, int64_t C, int64_t S, int ntn, const float* __restrict__ probs,
    const int* __restrict__ idx, const int* __restrict__ rank, const uint8_t* __restrict__ drop,
    const float* __restrict__ gate, const float* __restrict__ dgp,
    const int* __restrict__ counts1, float loss_scale, float* __restrict__ dh,
    __nv_bfloat16* __restrict__ dhp, __nv_bfloat16* __restrict__ dhs, float* __restrict__ dgate,
    int* __restrict__ drop_list, int* __restrict__ n_drop) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kWarpsPerBlock + warp;
  if (t >= T) return;
  bool kept[2];
  int e[2];
  int64_t s[2];
  float dg[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int64_t a = r * T + t;
    kept[r] = drop[a] == 0;
    e[r] = idx[a];
    s[r] = static_cast<int64_t>(e[r]) * C + rank[a];
    dg[r] = 0.f;
    if (kept[r]) {
      float sum = 0.f;
      for (int j = 0; j < ntn; ++j) sum += dgp[s[r] * ntn + j];     // fixed order
      // a gate that underflowed to 0 scaled dY to 0: its gradient is not
      // recoverable here, and p = 0 removes it from dh anyway
      const float g = gate[a];
      dg[r] = g > 0.f ? sum / g : 0.f;
    }
  }
  if (!kept[0] && !kept[1] && lane == 0) drop_list[atomicAdd(n_drop, 1)] = static_cast<int>(t);
  auto dp_of = [&](int i) {
    float v = loss_scale * static_cast<float>(counts1[i]);
    if (kept[0] && i == e[0]) v += dg[0];
    if (kept[1] && i == e[1]) v += dg[1];
    return v;
  };
  const float* prow = probs + t * N;
  float acc = 0.f;
  for (int i = lane; i < N; i += 32) acc = fmaf(prow[i], dp_of(i), acc);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  __syncwarp();
  const int64_t s_main = kept[0] ? s[0] : s[1];           // carries the router term
  const bool second = kept[0] && kept[1];                 // s[1] gets zero planes
  const __nv_bfloat16 zero = __float2bfloat16_rn(0.f);
  for (int i = lane; i < Np; i += 32) {
    float v = 0.f;
    if (i < N) {
      v = prow[i] * (dp_of(i) - acc);
      dh[t * N + i] = v;
    }
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
    dhp[t * Np + i] = hi;
    dhp[T * Np + t * Np + i] = lo;
    if (kept[0] || kept[1]) {
      dhs[s_main * Np + i] = hi;
      dhs[S * Np + s_main * Np + i] = lo;
    }
    if (second) {
      dhs[s[1] * Np + i] = zero;
      dhs[S * Np + s[1] * Np + i] = zero;
    }
  }
  if (dgate != nullptr && lane == 0) {
    dgate[t] = dg[0];
    dgate[T + t] = dg[1];
  }
}

// One warp per token (top-2): dx[t] = bf16(residual + dxs[s_0] + dxs[s_1])
// over the kept routes, in route order; tokens with no kept route are left
// to the dropped-token kernel.
__global__ void __launch_bounds__(256) bwd_combine_top2_kernel(
    int64_t T, int d, int64_t C, const int* __restrict__ idx, const int* __restrict__ rank,
    const uint8_t* __restrict__ drop, const float4* __restrict__ dxs,
    const uint4* __restrict__ dout, uint4* __restrict__ dx, int residual) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kWarpsPerBlock + warp;
  if (t >= T) return;
  const bool k0 = drop[t] == 0, k1 = drop[T + t] == 0;
  if (!k0 && !k1) return;
  const int64_t s0 = static_cast<int64_t>(idx[t]) * C + rank[t];
  const int64_t s1 = static_cast<int64_t>(idx[T + t]) * C + rank[T + t];
  const int dv = d / 8;                  // 8 bf16 per uint4, two float4 of dxs
  for (int v = lane; v < dv; v += 32) {
    float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (residual) {
      const uint4 g = __ldg(dout + t * dv + v);
      const uint32_t w[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        a[2 * j] = bf16_lo(w[j]);
        a[2 * j + 1] = bf16_hi(w[j]);
      }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      if (!(r == 0 ? k0 : k1)) continue;
      const float4* src = dxs + (r == 0 ? s0 : s1) * (d / 4) + 2 * v;
      const float4 u0 = __ldg(src), u1 = __ldg(src + 1);
      a[0] += u0.x; a[1] += u0.y; a[2] += u0.z; a[3] += u0.w;
      a[4] += u1.x; a[5] += u1.y; a[6] += u1.z; a[7] += u1.w;
    }
    dx[t * dv + v] = make_uint4(pack_bf16x2(a[0], a[1]), pack_bf16x2(a[2], a[3]),
                                pack_bf16x2(a[4], a[5]), pack_bf16x2(a[6], a[7]));
  }
}

// wrp[0][i][k] = bf16(W_r[i, k]), wrp[1][i][k] = bf16(W_r[i, k] - hi), zero
// rows for N <= i < Np.
__global__ void wr_split_kernel(int N, int Np, int d, const float* __restrict__ w_r,
                                __nv_bfloat16* __restrict__ wrp) {
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t n = static_cast<int64_t>(Np) * d;
  if (j >= n) return;
  const float w = j < static_cast<int64_t>(N) * d ? w_r[j] : 0.f;
  const __nv_bfloat16 hi = __float2bfloat16_rn(w);
  wrp[j] = hi;
  wrp[n + j] = __float2bfloat16_rn(w - __bfloat162float(hi));
}

constexpr int kDropTok = 16;     // dropped tokens per block

// dx[t] = (residual ? dout[t] : 0) + dh[t] . W_r for the listed tokens;
// block (b, y) takes list entries [16 g, 16 g + 16) for g = b, b + gridDim.x,
// ... and columns [256 y, 256 y + 256): dh rows staged in shared memory,
// each W_r element read once per group.
__global__ void __launch_bounds__(256) bwd_dropped_kernel(
    int N, int d, const int* __restrict__ drop_list, const int* __restrict__ n_drop,
    const float* __restrict__ dh, const float* __restrict__ w_r,
    const __nv_bfloat16* __restrict__ dout, __nv_bfloat16* __restrict__ dx, int residual) {
  extern __shared__ float sdh[];                       // [kDropTok][N]
  __shared__ int toks[kDropTok];
  const int nd = *n_drop;
  for (int first = blockIdx.x * kDropTok; first < nd; first += gridDim.x * kDropTok) {
    const int cnt = nd - first < kDropTok ? nd - first : kDropTok;
    __syncthreads();                                     // previous group done with sdh / toks
    if (threadIdx.x < kDropTok) toks[threadIdx.x] = threadIdx.x < cnt ? drop_list[first + threadIdx.x] : -1;
    __syncthreads();
    for (int q = threadIdx.x; q < kDropTok * N; q += blockDim.x) {
      const int j = q / N, i = q - j * N;
      sdh[q] = j < cnt ? dh[static_cast<int64_t>(toks[j]) * N + i] : 0.f;
    }
    __syncthreads();
    for (int k = blockIdx.y * blockDim.x + threadIdx.x; k < d; k += gridDim.y * blockDim.x) {
      float acc[kDropTok];
#pragma unroll
      for (int j = 0; j < kDropTok; ++j) acc[j] = 0.f;
      int i = 0;
      for (; i + 16 <= N; i += 16) {        // sixteen W_r loads in flight
        float w[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) w[u] = __ldg(w_r + static_cast<int64_t>(i + u) * d + k);
#pragma unroll
        for (int u = 0; u < 16; ++u)
#pragma unroll
          for (int j = 0; j < kDropTok; ++j) acc[j] = fmaf(sdh[j * N + i + u], w[u], acc[j]);
      }
      for (; i < N; ++i) {
        const float w = __ldg(w_r + static_cast<int64_t>(i) * d + k);
#pragma unroll
        for (int j = 0; j < kDropTok; ++j) acc[j] = fmaf(sdh[j * N + i], w, acc[j]);
      }
      for (int j = 0; j < cnt; ++j) {
        const int64_t o = static_cast<int64_t>(toks[j]) * d + k;
        const float r = residual ? __bfloat162float(dout[o]) : 0.f;
        dx[o] = __float2bfloat16_rn(r + acc[j]);
      }
    }
  }
}

unsigned warp_blocks(int64_t rows) {
  return static_cast<unsigned>((rows + kWarpsPerBlock - 1) / kWarpsPerBlock);
}

}  // namespace

cudaError_t launch_bwd_gather(int64_t C, int N, int d, int F, const int* counts,
                              const int* slot_token, const float* gate, const int* idx,
                              int64_t T2, const void* dout, void* dys, void* hbuf,
                              cudaStream_t st) {
  const int64_t S = static_cast<int64_t>(N) * C;
  if (S == 0) return cudaSuccess;
  bwd_gather_kernel<<<warp_blocks(S), 256, 0, st>>>(
      S, C, d, F, counts, slot_token, gate, idx, T2, static_cast<const uint4*>(dout),
      static_cast<uint4*>(dys), static_cast<uint4*>(hbuf));
  return cudaGetLastError();
}

cudaError_t launch_router_bwd_dh(int64_t T, int N, int Np, int64_t C, int ntn,
                                 const float* probs, const int* idx, const int* rank,
                                 const uint8_t* drop, const float* gate, const float* dgp,
                                 const int* counts, float loss_scale, float* dh, void* dhp,
                                 void* dhs, float* dgate, int* drop_list, int* n_drop,
                                 cudaStream_t st) {
  const int64_t S = static_cast<int64_t>(N) * C;
  router_bwd_dh_kernel<<<warp_blocks(T), 256, 0, st>>>(
      T, N, Np, C, S, ntn, probs, idx, rank, drop, gate, dgp, counts, loss_scale, dh,
      static_cast<__nv_bfloat16*>(dhp), static_cast<__nv_bfloat16*>(dhs), dgate, drop_list,
      n_drop);
  return cudaGetLastError();
}

cudaError_t launch_router_bwd_dh_top2(int64_t T, int N, int Np, int64_t C, int ntn,
                                      const float* probs, const int* idx, const int* rank,
                                      const uint8_t* drop, const float* gate, const float* dgp,
                                      const int* counts1, float loss_scale, float* dh,
                                      void* dhp, void* dhs, float* dgate, int* drop_list,
                                      int* n_drop, cudaStream_t st) {
  const int64_t S = static_cast<int64_t>(N) * C;
  router_bwd_dh_top2_kernel<<<warp_blocks(T), 256, 0, st>>>(
      T, N, Np, C, S, ntn, probs, idx, rank, drop, gate, dgp, counts1, loss_scale, dh,
      static_cast<__nv_bfloat16*>(dhp), static_cast<__nv_bfloat16*>(dhs), dgate, drop_list,
      n_drop);
  return cudaGetLastError();
}

cudaError_t launch_bwd_combine_top2(int64_t T, int d, int64_t C, const int* idx, const int* rank,
                                    const uint8_t* drop, const float* dxs, const void* dout,
                                    void* dx, bool residual, cudaStream_t st) {
  bwd_combine_top2_kernel<<<warp_blocks(T), 256, 0, st>>>(
      T, d, C, idx, rank, drop, reinterpret_cast<const float4*>(dxs),
      static_cast<const uint4*>(dout), static_cast<uint4*>(dx), residual ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_wr_split(int N, int d, const float* w_r, void* wrp, cudaStream_t st) {
  const int Np = (N + 63) / 64 * 64;
  const int64_t n = static_cast<int64_t>(Np) * d;
  wr_split_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(
      N, Np, d, w_r, static_cast<__nv_bfloat16*>(wrp));
  return cudaGetLastError();
}

cudaError_t launch_bwd_dropped(int64_t T, int N, int d, const int* drop_list, const int* n_drop,
                               const float* dh, const float* w_r, const void* dout, void* dx,
                               bool residual, cudaStream_t st) {
  const size_t smem = sizeof(float) * kDropTok * static_cast<size_t>(N);
  static size_t smem_set[64] = {};
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(&bwd_dropped_kernel), smem,
                                    smem_set);
  if (e != cudaSuccess) return e;
  // a few waves at most: blocks loop over the list in steps of the grid
  const int64_t groups = (T + kDropTok - 1) / kDropTok;
  const dim3 blocks(static_cast<unsigned>(groups < 296 ? groups : 296),
                    static_cast<unsigned>((d + 255) / 256));
  bwd_dropped_kernel<<<blocks, 256, smem, st>>>(
      N, d, drop_list, n_drop, dh, w_r, static_cast<const __nv_bfloat16*>(dout),
      static_cast<__nv_bfloat16*>(dx), residual ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace smoe
