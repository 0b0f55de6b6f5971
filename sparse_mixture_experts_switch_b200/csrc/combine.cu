// Combine and load-balancing loss.
//
// Combine: "Switch Transformers: scaling to trillion-parameter models",
// section "Switch Routing: From Top-k to k = 1", combine equation
// y = sum over the selected set of p_i(x) E_i(x) (one expert, or two with
// top-2 routing); a dropped assignment contributes nothing and a token with
// none left is its residual (section "Expert Capacity and the Capacity
// Factor").
// Loss: section "The Load-Balancing Loss", alpha . N . sum_i f_i P_i.
#include "kernels.cuh"

namespace smoe {

// ------------------------------------------------------------------ combine

template <bool kBF16>
__global__ void __launch_bounds__(256) combine_kernel(
    int64_t T, int vec_per_row, int64_t C, const uint4* __restrict__ x,
    const int* __restrict__ idx, const int* __restrict__ rank,
    const uint8_t* __restrict__ drop, const float* __restrict__ gate,
    const uint4* __restrict__ y, uint4* __restrict__ out, bool only_dropped, int routes) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       t < T; t += warps) {
    // route r of token t is entry r * T + t (routes <= 2)
    const bool dropped = drop[t] != 0;
    if (only_dropped && !dropped) continue;
    float g[2];
    const uint4* yrow[2];
    for (int r = 0; r < 2; ++r) {
      const int64_t a = r * T + t;
      const bool here = r < routes && drop[a] == 0;
      g[r] = here ? gate[a] : 0.f;
      yrow[r] = here ? y + (static_cast<int64_t>(idx[a]) * C + rank[a]) * vec_per_row : nullptr;
    }
    const uint4* xrow = x ? x + t * vec_per_row : nullptr;
    uint4* orow = out + t * vec_per_row;
    if (yrow[0] == nullptr && yrow[1] == nullptr) {
      // nothing kept: the residual row as it is (bit for bit, -0 included)
      for (int v = lane; v < vec_per_row; v += 32)
        orow[v] = xrow ? __ldg(xrow + v) : make_uint4(0, 0, 0, 0);
      continue;
    }
    for (int v = lane; v < vec_per_row; v += 32) {
      const uint4 xv = xrow ? __ldg(xrow + v) : make_uint4(0, 0, 0, 0);
      const uint4 y0 = yrow[0] ? __ldg(yrow[0] + v) : make_uint4(0, 0, 0, 0);
      const uint4 y1 = yrow[1] ? __ldg(yrow[1] + v) : make_uint4(0, 0, 0, 0);
      uint4 o;
      if (kBF16) {
        const uint32_t* xa = &xv.x;
        const uint32_t* ya = &y0.x;
        const uint32_t* yb = &y1.x;
        uint32_t* oa = &o.x;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float lo = fmaf(g[1], bf16_lo(yb[i]), fmaf(g[0], bf16_lo(ya[i]), bf16_lo(xa[i])));
          const float hi = fmaf(g[1], bf16_hi(yb[i]), fmaf(g[0], bf16_hi(ya[i]), bf16_hi(xa[i])));
          oa[i] = pack_bf16x2(lo, hi);
        }
      } else {
        const float* xa = reinterpret_cast<const float*>(&xv);
        const float* ya = reinterpret_cast<const float*>(&y0);
        const float* yb = reinterpret_cast<const float*>(&y1);
        float* oa = reinterpret_cast<float*>(&o);
#pragma unroll
        for (int i = 0; i < 4; ++i) oa[i] = fmaf(g[1], yb[i], fmaf(g[0], ya[i], xa[i]));
      }
      orow[v] = o;
    }
  }
}

cudaError_t launch_combine(int64_t T, int d, int64_t C, bool bf16, const void* x,
                           const int* idx, const int* rank, const uint8_t* drop,
                           const float* gate, const void* y, void* out, bool only_dropped,
                           int routes, cudaStream_t st) {
  const int vec = d * (bf16 ? 2 : 4) / 16;
  int64_t blocks = (T + 7) / 8;
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks < 1) blocks = 1;
  if (bf16)
    combine_kernel<true><<<static_cast<int>(blocks), 256, 0, st>>>(
        T, vec, C, static_cast<const uint4*>(x), idx, rank, drop, gate,
        static_cast<const uint4*>(y), static_cast<uint4*>(out), only_dropped, routes);
  else
    combine_kernel<false><<<static_cast<int>(blocks), 256, 0, st>>>(
        T, vec, C, static_cast<const uint4*>(x), idx, rank, drop, gate,
        static_cast<const uint4*>(y), static_cast<uint4*>(out), only_dropped, routes);
  return cudaGetLastError();
}

// --------------------------------------------------------------- aux loss

// psum[blk][e] = sum over rows blk*128 .. blk*128+127 of probs[row][e], in a
// fixed order.  One block per 128-row part; a thread owns one column unit (4
// experts as a float4 when N % 4 == 0, else one expert) and one of G row
// groups (rows g, g + G, ...), so a warp reads whole row segments and every
// thread keeps several independent loads in flight; the G partial sums of a
// unit are then added in group order.
template <bool kVec4>
__device__ __forceinline__ void colsum_part(int64_t T, int N, const float* __restrict__ probs,
                                            float* __restrict__ psum, float4* red) {
  const int units = kVec4 ? N / 4 : N;
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * kTileTok;
  const int rows = static_cast<int>(T - r0 < kTileTok ? T - r0 : kTileTok);
  for (int u0 = 0; u0 < units; u0 += 256) {
    const int span = units - u0 < 256 ? units - u0 : 256;   // units in this pass
    const int G = 256 / span;                                // row groups
    const int u = u0 + static_cast<int>(threadIdx.x) % span;
    const int g = static_cast<int>(threadIdx.x) / span;
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    if (g < G) {
      if (kVec4) {
        const float4* col = reinterpret_cast<const float4*>(probs + r0 * N) + u;
        // up to 16 rows' loads in flight per thread, then added in row order
        for (int r0 = g; r0 < rows; r0 += 16 * G) {
          float4 v[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const int r = r0 + k * G;
            v[k] = r < rows ? __ldg(col + static_cast<int64_t>(r) * (N / 4))
                            : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            s.x += v[k].x; s.y += v[k].y; s.z += v[k].z; s.w += v[k].w;
          }
        }
      } else {
        const float* col = probs + r0 * N + u;
        for (int r0 = g; r0 < rows; r0 += 16 * G) {
          float v[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const int r = r0 + k * G;
            v[k] = r < rows ? __ldg(col + static_cast<int64_t>(r) * N) : 0.f;
          }
#pragma unroll
          for (int k = 0; k < 16; ++k) s.x += v[k];
        }
      }
    }
    red[threadIdx.x] = s;
    __syncthreads();
    if (static_cast<int>(threadIdx.x) < span) {
      float4 t = red[threadIdx.x];
      for (int q = 1; q < G; ++q) {
        const float4 v = red[q * span + threadIdx.x];
        t.x += v.x; t.y += v.y; t.z += v.z; t.w += v.w;
      }
      float* dst = psum + static_cast<int64_t>(blockIdx.x) * N;
      if (kVec4) reinterpret_cast<float4*>(dst)[u] = t;
      else dst[u] = t.x;
    }
    __syncthreads();
  }
}

template <bool kVec4>
__global__ void __launch_bounds__(256) prob_colsum_kernel(int64_t T, int N,
                                                          const float* __restrict__ probs,
                                                          float* __restrict__ psum) {
  __shared__ float4 red[256];
  colsum_part<kVec4>(T, N, probs, psum, red);
}

cudaError_t launch_prob_colsum(int64_t T, int N, const float* probs, float* psum,
                               cudaStream_t st) {
  const unsigned grid = static_cast<unsigned>((T + kTileTok - 1) / kTileTok);
  const bool vec4 = (N % 4) == 0 && (reinterpret_cast<uintptr_t>(probs) & 15u) == 0 &&
                    (reinterpret_cast<uintptr_t>(psum) & 15u) == 0;
  if (vec4)
    prob_colsum_kernel<true><<<grid, 256, 0, st>>>(T, N, probs, psum);
  else
    prob_colsum_kernel<false><<<grid, 256, 0, st>>>(T, N, probs, psum);
  return cudaGetLastError();
}

// Two fixed-order stages in one launch.  Block (bx, by) owns experts
// [32 bx, 32 bx + 32) and the by-th of kAuxChunks equal runs of parts: its 8
// warps split the run, each lane one expert, partial sums in double, the
// warps' sums added in warp order into part_sum[by][e].  The last block to
// finish (a ticket counter decides only *which* block, not any order of
// additions) adds the runs in order, forms f_e P_e and sums over experts in
// a fixed tree.
__global__ void __launch_bounds__(256) aux_loss_kernel(int64_t T, int N, int nparts,
                                                       float alpha,
                                                       const int* __restrict__ counts,
                                                       const float* __restrict__ psum,
                                                       float* __restrict__ loss,
                                                       float* __restrict__ f_out,
                                                       float* __restrict__ P_out,
                                                       double* __restrict__ part_sum,
                                                       unsigned* __restrict__ ticket) {
  __shared__ double part[8][32];
  __shared__ double red[256];
  __shared__ bool last;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x * 32 + lane;
  const int per = (nparts + gridDim.y - 1) / gridDim.y;
  const int p0 = blockIdx.y * per;
  const int p1 = p0 + per < nparts ? p0 + per : nparts;
  double s = 0.0;
  if (e < N)
    for (int pp = p0 + w; pp < p1; pp += 8)
      s += static_cast<double>(psum[static_cast<int64_t>(pp) * N + e]);
  part[w][lane] = s;
  __syncthreads();
  if (w == 0 && e < N) {
    double tot = 0.0;
    for (int q = 0; q < 8; ++q) tot += part[q][lane];
    part_sum[static_cast<int64_t>(blockIdx.y) * N + e] = tot;
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last = atomicAdd(ticket, 1u) == gridDim.x * gridDim.y - 1;
  __syncthreads();
  if (!last) return;
  __threadfence();
  double acc = 0.0;
  for (int i = threadIdx.x; i < N; i += 256) {
    double tot = 0.0;
    for (unsigned c = 0; c < gridDim.y; ++c)
      tot += const_cast<volatile double*>(part_sum)[static_cast<int64_t>(c) * N + i];
    const double P = tot / static_cast<double>(T);
    const double f = static_cast<double>(counts[i]) / static_cast<double>(T);
    if (f_out) f_out[i] = static_cast<float>(f);
    if (P_out) P_out[i] = static_cast<float>(P);
    acc += f * P;
  }
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int st = 128; st > 0; st >>= 1) {
    if (threadIdx.x < st) red[threadIdx.x] += red[threadIdx.x + st];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    if (loss) *loss = static_cast<float>(static_cast<double>(alpha) * N * red[0]);
    *ticket = 0;                 // ready for the next call on this workspace
  }
}

cudaError_t launch_aux_loss(int64_t T, int N, int nparts, float alpha, const int* counts,
                            const float* psum, float* loss, float* f, float* P,
                            double* part_sum, unsigned* ticket, cudaStream_t st) {
  const int chunks = nparts < kAuxChunks ? (nparts > 0 ? nparts : 1) : kAuxChunks;
  const dim3 grid(static_cast<unsigned>((N + 31) / 32), static_cast<unsigned>(chunks));
  aux_loss_kernel<<<grid, 256, 0, st>>>(T, N, nparts, alpha, counts, psum, loss, f, P,
                                        part_sum, ticket);
  return cudaGetLastError();
}

// The staged loss from full probabilities in one launch: block b sums part b
// (128 rows, fixed order) into psum[b]; the last block of each of the
// kAuxChunks runs of parts (a per-run ticket picks which block, not any
// order of additions) adds the run's parts in order in double into
// part_sum[run]; the last run to finish forms f_e P_e and the loss in a
// fixed tree.  Tickets are left at zero for the next call.
template <bool kVec4>
__global__ void __launch_bounds__(256) aux_loss_probs_kernel(
    int64_t T, int N, float alpha, const int* __restrict__ counts,
    const float* __restrict__ probs, float* __restrict__ psum, float* __restrict__ loss,
    float* __restrict__ f_out, float* __restrict__ P_out, double* __restrict__ part_sum,
    unsigned* __restrict__ run_ticket, unsigned* __restrict__ ticket) {
  __shared__ float4 red4[256];
  __shared__ double red[256];
  __shared__ bool last;
  colsum_part<kVec4>(T, N, probs, psum, red4);
  const int nparts = static_cast<int>(gridDim.x);
  const int per = (nparts + kAuxChunks - 1) / kAuxChunks;   // parts per run
  const int nruns = (nparts + per - 1) / per;                // runs that hold parts
  const int run = static_cast<int>(blockIdx.x) / per;
  const int p0 = run * per;
  const int p1 = p0 + per < nparts ? p0 + per : nparts;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last = atomicAdd(&run_ticket[run], 1u) == static_cast<unsigned>(p1 - p0 - 1);
  __syncthreads();
  if (!last) return;
  __threadfence();
  for (int e = threadIdx.x; e < N; e += 256) {
    // 16 parts' loads in flight at a time, added in part order
    double tot = 0.0;
    for (int pb = p0; pb < p1; pb += 16) {
      float v[16];
#pragma unroll
      for (int j = 0; j < 16; ++j)
        v[j] = pb + j < p1 ? __ldcg(psum + static_cast<int64_t>(pb + j) * N + e) : 0.f;
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (pb + j < p1) tot += static_cast<double>(v[j]);
    }
    part_sum[static_cast<int64_t>(run) * N + e] = tot;
  }
  if (threadIdx.x == 0) run_ticket[run] = 0;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last = atomicAdd(ticket, 1u) == static_cast<unsigned>(nruns - 1);
  __syncthreads();
  if (!last) return;
  __threadfence();
  double acc = 0.0;
  for (int i = threadIdx.x; i < N; i += 256) {
    double v[kAuxChunks];                 // every run's sum in flight, added in run order
#pragma unroll
    for (int c = 0; c < kAuxChunks; ++c)
      v[c] = c < nruns ? __ldcg(part_sum + static_cast<int64_t>(c) * N + i) : 0.0;
    double tot = 0.0;
#pragma unroll
    for (int c = 0; c < kAuxChunks; ++c)
      if (c < nruns) tot += v[c];
    const double P = tot / static_cast<double>(T);
    const double f = static_cast<double>(counts[i]) / static_cast<double>(T);
    if (f_out) f_out[i] = static_cast<float>(f);
    if (P_out) P_out[i] = static_cast<float>(P);
    acc += f * P;
  }
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int st = 128; st > 0; st >>= 1) {
    if (threadIdx.x < st) red[threadIdx.x] += red[threadIdx.x + st];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    if (loss) *loss = static_cast<float>(static_cast<double>(alpha) * N * red[0]);
    *ticket = 0;
  }
}

cudaError_t launch_aux_loss_probs(int64_t T, int N, float alpha, const int* counts,
                                  const float* probs, float* psum, float* loss, float* f,
                                  float* P, double* part_sum, unsigned* run_ticket,
                                  unsigned* ticket, cudaStream_t st) {
  const unsigned grid = static_cast<unsigned>((T + kTileTok - 1) / kTileTok);
  const bool vec4 = (N % 4) == 0 && (reinterpret_cast<uintptr_t>(probs) & 15u) == 0 &&
                    (reinterpret_cast<uintptr_t>(psum) & 15u) == 0;
  if (vec4)
    aux_loss_probs_kernel<true><<<grid, 256, 0, st>>>(T, N, alpha, counts, probs, psum, loss, f,
                                                       P, part_sum, run_ticket, ticket);
  else
    aux_loss_probs_kernel<false><<<grid, 256, 0, st>>>(T, N, alpha, counts, probs, psum, loss, f,
                                                        P, part_sum, run_ticket, ticket);
  return cudaGetLastError();
}

}  // namespace smoe
