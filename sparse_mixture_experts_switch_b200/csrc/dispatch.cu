// Capacity-bounded dispatch ("Switch Transformers: scaling to
// trillion-parameter models", section "Expert Capacity and the Capacity
// Factor": each expert has C slots; tokens beyond C are dropped and pass
// through on the residual; unused slots are padding).
//
// Slot order is batch order.  It is computed without any atomic that could
// reorder slots:
//   1. per 128-token tile, each warp ranks its tokens with __match_any_sync
//      (lanes with the same expert) and a popcount of the lower lanes; the
//      four warps' counts are offset in warp order -> rank within the tile,
//      and the tile's per-expert histogram;
//   2. an exclusive scan of every expert's histogram down the tile axis;
//   3. rank = scanned base + rank within the tile; drop = rank >= C.
#include "kernels.cuh"

namespace smoe {

__global__ void __launch_bounds__(kTileTok) tile_rank_kernel(
    int64_t T, int N, const int* __restrict__ idx_in, const float* __restrict__ probs,
    int* __restrict__ idx_out, int* __restrict__ local_rank, int* __restrict__ hist,
    int ntiles, DevErr* err) {
  extern __shared__ int cnt[];   // [4][N]
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.x;
  for (int i = tid; i < 4 * N; i += kTileTok) cnt[i] = 0;
  __syncthreads();

  const int64_t t = static_cast<int64_t>(tile) * kTileTok + tid;
  int e = -1;
  if (t < T) {
    if (idx_in != nullptr) {
      e = idx_in[t];
    } else {
      const float* row = probs + t * N;
      float best = row[0];
      e = 0;
      for (int j = 1; j < N; ++j) {
        const float v = row[j];
        if (v > best) { best = v; e = j; }
      }
    }
    if (e < 0 || e >= N) {
      report_error(err, SWITCH_ERR_DEVICE_BOUNDS, kWhereDispatch, t);
      e = -1;
    }
  }
  const unsigned peers = __match_any_sync(0xffffffffu, e);
  const int rank_w = __popc(peers & ((1u << lane) - 1u));
  if (e >= 0 && rank_w == 0) cnt[w * N + e] = __popc(peers);
  __syncthreads();
  if (t < T) {
    int r = -1;
    if (e >= 0) {
      r = rank_w;
      for (int q = 0; q < w; ++q) r += cnt[q * N + e];
    }
    local_rank[t] = r;
    if (idx_out != nullptr) idx_out[t] = e;
  }
  for (int j = tid; j < N; j += kTileTok)
    hist[static_cast<int64_t>(j) * ntiles + tile] =
        cnt[j] + cnt[N + j] + cnt[2 * N + j] + cnt[3 * N + j];
}

cudaError_t launch_tile_rank(int64_t T, int N, const int* idx_in, const float* probs,
                             int* idx_out, int* local_rank, int* hist, int ntiles,
                             DevErr* err, cudaStream_t st) {
  const size_t sm = sizeof(int) * 4 * N;
  tile_rank_kernel<<<ntiles, kTileTok, sm, st>>>(T, N, idx_in, probs, idx_out, local_rank,
                                                 hist, ntiles, err);
  return cudaGetLastError();
}

// One block per expert: exclusive scan over its ntiles histogram entries.
// With a loss (ScanLoss::loss set), each block then also forms its expert's
// f_e P_e from the router's per-part probability sums, and the last block
// to finish (a ticket picks which block, not any order of additions) adds
// them into the loss: the additions are those of aux_loss_kernel, in the
// same order, so both give the same bits.
__global__ void __launch_bounds__(256) scan_kernel(int ntiles, const int* __restrict__ hist,
                                                   int* __restrict__ base,
                                                   int* __restrict__ counts, ScanLoss L) {
  __shared__ int warp_tot[8];
  __shared__ double cpart[kAuxChunks][8];
  __shared__ double red[256];
  __shared__ bool last;
  const int e = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int* h = hist + static_cast<int64_t>(e) * ntiles;
  int* b = base + static_cast<int64_t>(e) * ntiles;
  int carry = 0;
  for (int c0 = 0; c0 < ntiles; c0 += 256 * 4) {
    int v[4];
    int s = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int j = c0 + tid * 4 + i;
      v[i] = j < ntiles ? h[j] : 0;
      s += v[i];
    }
    // inclusive scan of the per-thread sums within the warp
    int inc = s;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, inc, off);
      if (lane >= off) inc += n;
    }
    if (lane == 31) warp_tot[w] = inc;
    __syncthreads();
    int woff = 0, total = 0;
    for (int q = 0; q < 8; ++q) {
      if (q < w) woff += warp_tot[q];
      total += warp_tot[q];
    }
    int run = carry + woff + inc - s;   // exclusive prefix of this thread
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int j = c0 + tid * 4 + i;
      if (j < ntiles) b[j] = run;
      run += v[i];
    }
    carry += total;
    __syncthreads();
  }
  if (tid == 0) counts[e] = carry;
  if (L.loss == nullptr) return;

  // P_e: chunk `by` of the parts, warp lane w of it (parts p0 + w, + 8, ...)
  const int N = static_cast<int>(gridDim.x);
  const int chunks = L.nparts < kAuxChunks ? (L.nparts > 0 ? L.nparts : 1) : kAuxChunks;
  const int per = (L.nparts + chunks - 1) / chunks;
  if (tid < chunks * 8) {
    const int by = tid >> 3, wq = tid & 7;
    const int p0 = by * per;
    const int p1 = p0 + per < L.nparts ? p0 + per : L.nparts;
    double sp = 0.0;
    for (int pp = p0 + wq; pp < p1; pp += 8)
      sp += static_cast<double>(L.psum[static_cast<int64_t>(pp) * N + e]);
    cpart[by][wq] = sp;
  }
  __syncthreads();
  if (tid == 0) {
    double tot = 0.0;
    for (int by = 0; by < chunks; ++by) {
      double part = 0.0;
      for (int q = 0; q < 8; ++q) part += cpart[by][q];
      tot += part;
    }
    const double P = tot / static_cast<double>(L.T);
    const double f = static_cast<double>(carry) / static_cast<double>(L.T);
    L.fp[e] = f * P;
    __threadfence();
    last = atomicAdd(L.ticket, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (!last) return;
  __threadfence();
  double acc = 0.0;
  for (int i = tid; i < N; i += 256) acc += __ldcg(L.fp + i);
  red[tid] = acc;
  __syncthreads();
  for (int stp = 128; stp > 0; stp >>= 1) {
    if (tid < stp) red[tid] += red[tid + stp];
    __syncthreads();
  }
  if (tid == 0) {
    *L.loss = static_cast<float>(static_cast<double>(L.alpha) * N * red[0]);
    *L.ticket = 0;               // ready for the next call on this workspace
  }
}

cudaError_t launch_scan(int N, int ntiles, const int* hist, int* base, int* counts,
                        cudaStream_t st, const ScanLoss* loss) {
  ScanLoss L{};
  if (loss != nullptr) L = *loss;
  scan_kernel<<<N, 256, 0, st>>>(ntiles, hist, base, counts, L);
  return cudaGetLastError();
}

// Per-expert number of 128-row M tiles, ceil(min(count, C) / 128), and its
// exclusive prefix (one warp).
__device__ void mtile_prefix_warp(int N, int64_t C, const int* __restrict__ counts,
                                  int* __restrict__ mtile_start) {
  const int lane = threadIdx.x & 31;
  const int per = (N + 31) / 32;
  int s = 0;
  for (int i = 0; i < per; ++i) {
    const int e = lane * per + i;
    if (e < N) {
      const int64_t kept = counts[e] < C ? counts[e] : C;
      s += static_cast<int>((kept + 127) / 128);
    }
  }
  int inc = s;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, inc, off);
    if (lane >= off) inc += n;
  }
  int run = inc - s;
  for (int i = 0; i < per; ++i) {
    const int e = lane * per + i;
    if (e < N) {
      mtile_start[e] = run;
      const int64_t kept = counts[e] < C ? counts[e] : C;
      run += static_cast<int>((kept + 127) / 128);
    }
  }
  if (lane == 31) mtile_start[N] = inc;
}

__global__ void __launch_bounds__(256) finalize_kernel(
    int64_t T, int N, int64_t C, int ntiles, const int* __restrict__ idx,
    const int* __restrict__ local_rank, const int* __restrict__ base,
    const int* __restrict__ counts, int* __restrict__ rank, uint8_t* __restrict__ drop,
    int* __restrict__ slot_token, int* __restrict__ mtile_start, int64_t tok_mod) {
  if (blockIdx.x == 0 && threadIdx.x < 32 && mtile_start != nullptr)
    mtile_prefix_warp(N, C, counts, mtile_start);
  const int64_t nslots = static_cast<int64_t>(N) * C;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
       i < (T > nslots ? T : nslots); i += stride) {
    if (i < T) {
      const int e = idx[i];
      const int lr = local_rank[i];
      int r = -1;
      bool dropped = true;
      if (e >= 0 && e < N && lr >= 0) {
        r = base[static_cast<int64_t>(e) * ntiles + (i / kTileTok)] + lr;
        dropped = r >= C;
        if (!dropped)
          slot_token[static_cast<int64_t>(e) * C + r] =
              static_cast<int>(tok_mod > 0 && i >= tok_mod ? i - tok_mod : i);
      }
      rank[i] = r;
      drop[i] = dropped ? 1 : 0;
    }
    if (i < nslots) {
      const int e = static_cast<int>(i / C);
      const int64_t r = i - static_cast<int64_t>(e) * C;
      const int64_t kept = counts[e] < C ? counts[e] : C;
      if (r >= kept) slot_token[i] = -1;
    }
  }
}

cudaError_t launch_finalize(int64_t T, int N, int64_t C, int ntiles, const int* idx,
                            const int* local_rank, const int* base, const int* counts,
                            int* rank, uint8_t* drop, int* slot_token, int* mtile_start,
                            int64_t tok_mod, cudaStream_t st) {
  const int64_t work = T > static_cast<int64_t>(N) * C ? T : static_cast<int64_t>(N) * C;
  int64_t blocks = (work + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks < 1) blocks = 1;
  finalize_kernel<<<static_cast<int>(blocks), 256, 0, st>>>(
      T, N, C, ntiles, idx, local_rank, base, counts, rank, drop, slot_token, mtile_start,
      tok_mod);
  return cudaGetLastError();
}

// finalize_kernel and the row copy in one pass.  Items 0 .. T-1 are
// assignments, items T .. T + N*C - 1 are slots.  A warp takes kGatherGroup
// consecutive items: lane j < kGatherGroup decides item j as finalize_kernel
// does (an assignment's rank, drop and slot; a padding slot's -1), so those
// metadata loads are in flight together; then the warp copies the items'
// rows one after another (16 bytes per lane per access): a kept token's row
// into its slot, zeros into a padding slot.  Groups are small so that many
// warps per SM each have a row in flight.  Without zero_pad the padding
// slots are not items at all (neither their rows nor their slot_token
// entries are written).  With `out` (top-1 layer, combine fused into the
// second GEMM) a dropped token's output row is written here as well: its
// residual x row (zeros without a residual), which is all the combine gives
// a token that no expert processed.
constexpr int kGatherGroup = 8;

__global__ void __launch_bounds__(256, 4) finalize_gather_kernel(
    int64_t T, int N, int64_t C, int ntiles, const int* __restrict__ idx,
    const int* __restrict__ local_rank, const int* __restrict__ base,
    const int* __restrict__ counts, int* __restrict__ rank, uint8_t* __restrict__ drop,
    int* __restrict__ slot_token, int* __restrict__ mtile_start, int64_t tok_mod,
    const uint4* __restrict__ x, uint4* __restrict__ x_disp, int64_t vec_per_row,
    uint4* __restrict__ out, bool out_residual, bool zero_pad) {
  if (blockIdx.x == 0 && threadIdx.x < 32 && mtile_start != nullptr)
    mtile_prefix_warp(N, C, counts, mtile_start);
  const int lane = threadIdx.x & 31;
  const int64_t nslots = static_cast<int64_t>(N) * C;
  // without zero_pad nothing reads the padding slots (their slot_token
  // entries included), so only the assignments are items
  const int64_t items = T + (zero_pad ? nslots : 0);
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t g0 = (static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5)) *
                    kGatherGroup;
       g0 < items; g0 += warps * kGatherGroup) {
    const int64_t i = lane < kGatherGroup ? g0 + lane : items;   // other lanes: no item
    int64_t dst = -1;        // x_disp row this lane's item writes
    int64_t src = -1;        // x row copied into it (-1: zeros)
    int64_t odst = -1;       // out row (a dropped token's) this item writes
    if (i < T) {
      const int e = idx[i];
      const int lr = local_rank[i];
      int r = -1;
      bool dropped = true;
      if (e >= 0 && e < N && lr >= 0) {
        r = base[static_cast<int64_t>(e) * ntiles + (i / kTileTok)] + lr;
        dropped = r >= C;
        if (!dropped) {
          const int64_t tok = tok_mod > 0 && i >= tok_mod ? i - tok_mod : i;
          dst = static_cast<int64_t>(e) * C + r;
          src = tok;
          slot_token[dst] = static_cast<int>(tok);
        }
      }
      if (dropped && out != nullptr) {
        odst = i;
        src = out_residual ? i : -1;
      }
      rank[i] = r;
      drop[i] = dropped ? 1 : 0;
    } else if (i < items) {
      const int64_t s = i - T;
      const int e = static_cast<int>(s / C);
      const int64_t r = s - static_cast<int64_t>(e) * C;
      const int64_t kept = counts[e] < C ? counts[e] : C;
      if (r >= kept) {             // (only with zero_pad: see `items`)
        slot_token[s] = -1;
        dst = s;
      }
    }
    // the group's rows side by side: every lane has one 16-byte load of each
    // row in flight before it stores any of them
    int d_j[kGatherGroup], s_j[kGatherGroup];          // row ids fit int32 (validated)
    const bool any_out = __any_sync(0xffffffffu, odst >= 0);
#pragma unroll
    for (int j = 0; j < kGatherGroup; ++j) {
      d_j[j] = __shfl_sync(0xffffffffu, static_cast<int>(dst), j);
      s_j[j] = __shfl_sync(0xffffffffu, static_cast<int>(src), j);
    }
    if (any_out) {
      // a dropped token among the group's items: one row at a time
      for (int j = 0; j < kGatherGroup; ++j) {
        const int o_j = __shfl_sync(0xffffffffu, static_cast<int>(odst), j);
        if (o_j < 0) continue;
        for (int64_t v = lane; v < vec_per_row; v += 32)
          out[static_cast<int64_t>(o_j) * vec_per_row + v] =
              s_j[j] >= 0 ? __ldg(x + static_cast<int64_t>(s_j[j]) * vec_per_row + v)
                          : make_uint4(0, 0, 0, 0);
      }
    }
    for (int64_t v = lane; v < vec_per_row; v += 32) {
      uint4 val[kGatherGroup];
#pragma unroll
      for (int j = 0; j < kGatherGroup; ++j)
        val[j] = (d_j[j] >= 0 && s_j[j] >= 0) ? __ldg(x + static_cast<int64_t>(s_j[j]) * vec_per_row + v)
                                              : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int j = 0; j < kGatherGroup; ++j)
        if (d_j[j] >= 0) x_disp[static_cast<int64_t>(d_j[j]) * vec_per_row + v] = val[j];
    }
  }
}

cudaError_t launch_finalize_gather(int64_t T, int N, int64_t C, int ntiles, const int* idx,
                                   const int* local_rank, const int* base, const int* counts,
                                   int* rank, uint8_t* drop, int* slot_token, int* mtile_start,
                                   int64_t tok_mod, const void* x, void* x_disp,
                                   int64_t row_bytes, cudaStream_t st, void* out,
                                   bool out_residual, bool zero_pad) {
  if (out != nullptr && tok_mod != 0) return cudaErrorInvalidValue;   // top-1 only
  const int64_t items = T + (zero_pad ? static_cast<int64_t>(N) * C : 0);
  int64_t blocks = (items + 8 * kGatherGroup - 1) / (8 * kGatherGroup);   // 8 warps a block
  if (blocks > 148 * 8) blocks = 148 * 8;
  if (blocks < 1) blocks = 1;
  finalize_gather_kernel<<<static_cast<int>(blocks), 256, 0, st>>>(
      T, N, C, ntiles, idx, local_rank, base, counts, rank, drop, slot_token, mtile_start,
      tok_mod, static_cast<const uint4*>(x), static_cast<uint4*>(x_disp), row_bytes / 16,
      static_cast<uint4*>(out), out_residual, zero_pad);
  return cudaGetLastError();
}

__global__ void mtile_table_kernel(int N, int64_t C, const int* counts, int* mtile_start) {
  mtile_prefix_warp(N, C, counts, mtile_start);
}

cudaError_t launch_mtile_table(int N, int64_t C, const int* counts, int* mtile_start,
                               cudaStream_t st) {
  mtile_table_kernel<<<1, 32, 0, st>>>(N, C, counts, mtile_start);
  return cudaGetLastError();
}

// One warp per slot row, 16-byte vectors.
__global__ void __launch_bounds__(256) gather_rows_kernel(int64_t nslots, int64_t vec_per_row,
                                                          const int* __restrict__ slot_token,
                                                          const uint4* __restrict__ x,
                                                          uint4* __restrict__ x_disp) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t s = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       s < nslots; s += warps) {
    const int tok = slot_token[s];
    uint4* dst = x_disp + s * vec_per_row;
    if (tok >= 0) {
      const uint4* src = x + static_cast<int64_t>(tok) * vec_per_row;
      for (int64_t v = lane; v < vec_per_row; v += 32) dst[v] = __ldg(src + v);
    } else {
      for (int64_t v = lane; v < vec_per_row; v += 32) dst[v] = make_uint4(0, 0, 0, 0);
    }
  }
}

cudaError_t launch_gather_rows(int64_t nslots, int64_t row_bytes, const int* slot_token,
                               const void* x, void* x_disp, cudaStream_t st) {
  if (nslots == 0) return cudaSuccess;
  int64_t blocks = (nslots + 7) / 8;
  if (blocks > 148 * 8) blocks = 148 * 8;
  gather_rows_kernel<<<static_cast<int>(blocks), 256, 0, st>>>(
      nslots, row_bytes / 16, slot_token, static_cast<const uint4*>(x),
      static_cast<uint4*>(x_disp));
  return cudaGetLastError();
}

}  // namespace smoe
