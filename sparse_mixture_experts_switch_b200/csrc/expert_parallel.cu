// Expert parallelism: the layer's experts spread over G ranks (GPUs), each
// rank holding N / G of them and its own T tokens ("Switch Transformers:
// scaling to trillion-parameter models", section "Distributed Implementation
// and the Three Parallelisms", expert-parallelism row: tokens travel to the
// device of their expert and back).
//
// The global batch is the ranks' batches end to end in rank order, one
// routing group, so capacity, drops and the loss are exactly those of one
// GPU holding all G T tokens:
//   * every rank routes its tokens and counts them per expert (router and
//     dispatch histograms, as on one GPU);
//   * the ranks all-gather (collective outside this file) one record each:
//     per-expert counts and per-128-token-part sums of the router
//     probabilities;
//   * a token's global rank within its expert is the count of the earlier
//     ranks' tokens on that expert plus its rank on its own rank (batch
//     order); it is dropped when that reaches C;
//   * ep_dispatch_kernel stores each kept token's row, its source (home rank,
//     token) and its gate straight into the owner's receive buffer through
//     peer pointers (plain stores over NVLink; no copy here reads another
//     GPU's memory, and none is a multicast);
//   * after a barrier, the owner runs the grouped GEMMs on its experts, and
//     the second GEMM's epilogue stores x + gate * E(x) into the home rank's
//     output row through a peer pointer (expert_ffn_pair.cu).
#include "kernels.cuh"

namespace smoe {

// Block 0: global counts (sum over ranks) and this rank's experts' counts.
// Every block: a share of the probability-sum parts copied end to end in
// rank order, [G * nparts][N].
__global__ void __launch_bounds__(256) ep_prepare_kernel(int N, int G, int me, int e_loc,
                                                         int nparts, EpGathered g,
                                                         int* __restrict__ counts_glob,
                                                         int* __restrict__ counts_loc,
                                                         float* __restrict__ psum_cat) {
  if (blockIdx.x == 0) {
    for (int e = threadIdx.x; e < N; e += blockDim.x) {
      int s = 0;
      for (int q = 0; q < G; ++q)
        s += reinterpret_cast<const int*>(g.base + q * g.stride + g.counts_off)[e];
      counts_glob[e] = s;
      if (e / e_loc == me) counts_loc[e - me * e_loc] = s;
    }
  }
  const int64_t per_rank = static_cast<int64_t>(nparts) * N;
  const int64_t total = per_rank * G;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t q = i / per_rank;
    psum_cat[i] = reinterpret_cast<const float*>(g.base + q * g.stride)[i - q * per_rank];
  }
}

cudaError_t launch_ep_prepare(int N, int G, int me, int e_loc, int nparts, EpGathered g,
                              int* counts_glob, int* counts_loc, float* psum_cat,
                              cudaStream_t st) {
  const int64_t total = static_cast<int64_t>(G) * nparts * N;
  int64_t blocks = (total + 255) / 256;
  if (blocks > 148 * 4) blocks = 148 * 4;
  if (blocks < 1) blocks = 1;
  ep_prepare_kernel<<<static_cast<int>(blocks), 256, 0, st>>>(N, G, me, e_loc, nparts, g,
                                                              counts_glob, counts_loc, psum_cat);
  return cudaGetLastError();
}

// One warp per token of rank r.  The earlier ranks' counts per expert are
// summed once per block into shared memory.
__global__ void __launch_bounds__(256) ep_dispatch_kernel(
    int64_t T, int N, int64_t C, int G, int r, int e_loc, int ntiles,
    const int* __restrict__ idx, const int* __restrict__ local_rank,
    const int* __restrict__ base, const float* __restrict__ gate, EpGathered g,
    const uint4* __restrict__ x, int64_t vec_per_row, EpPeers recv, EpRecvLayout rl,
    int* __restrict__ rank_out, uint8_t* __restrict__ drop_out) {
  extern __shared__ int before[];   // [N]: tokens of ranks 0 .. r-1 on each expert
  for (int e = threadIdx.x; e < N; e += blockDim.x) {
    int s = 0;
    for (int q = 0; q < r; ++q)
      s += reinterpret_cast<const int*>(g.base + q * g.stride + g.counts_off)[e];
    before[e] = s;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       t < T; t += warps) {
    const int e = idx[t];
    const int lr = local_rank[t];
    int64_t gr = -1;
    bool dropped = true;
    if (e >= 0 && e < N && lr >= 0) {
      gr = before[e] + static_cast<int64_t>(base[static_cast<int64_t>(e) * ntiles + t / kTileTok]) +
           lr;
      dropped = gr >= C;
    }
    if (lane == 0) {
      rank_out[t] = static_cast<int>(gr);
      drop_out[t] = dropped ? 1 : 0;
    }
    if (dropped) continue;
    const int h = e / e_loc;                                  // owner rank
    const int64_t slot = static_cast<int64_t>(e - h * e_loc) * C + gr;
    uint8_t* rb = static_cast<uint8_t*>(recv.p[h]);
    uint4* dst = reinterpret_cast<uint4*>(rb) + slot * vec_per_row;
    const uint4* src = x + t * vec_per_row;
    for (int64_t v = lane; v < vec_per_row; v += 32) dst[v] = __ldg(src + v);
    if (lane == 0) {
      reinterpret_cast<int*>(rb + rl.src_off)[slot] =
          (r << kEpRankShift) | static_cast<int>(t);
      reinterpret_cast<float*>(rb + rl.gate_off)[slot] = gate[t];
    }
  }
  // the stores above reach the owners before anything this rank signals later
  __threadfence_system();
}

cudaError_t launch_ep_dispatch(int64_t T, int N, int64_t C, int G, int r, int e_loc, int ntiles,
                               const int* idx, const int* local_rank, const int* base,
                               const float* gate, EpGathered g, const void* x, int64_t row_bytes,
                               const EpPeers& recv, EpRecvLayout rl, int* rank, uint8_t* drop,
                               cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  int64_t blocks = (T + 7) / 8;
  if (blocks > 148 * 8) blocks = 148 * 8;
  ep_dispatch_kernel<<<static_cast<int>(blocks), 256, sizeof(int) * N, st>>>(
      T, N, C, G, r, e_loc, ntiles, idx, local_rank, base, gate, g,
      static_cast<const uint4*>(x), row_bytes / 16, recv, rl, rank, drop);
  return cudaGetLastError();
}

}  // namespace smoe
