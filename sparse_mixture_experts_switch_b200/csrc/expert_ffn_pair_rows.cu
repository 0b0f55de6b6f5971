// Expert FFN GEMM on CTA pairs with the rows of the output as the MMA's M:
//
//   D[token r, f] = sum_k A[token r, k] * W[e][f, k]
//
// A pair tile is 256 of one expert's dispatched rows x 256 output columns.
// CTA q of the pair loads its own 128 rows of the dispatched buffer (the A
// operand) and 128 of the tile's 256 weight rows (its half of the B
// operand), both by TMA onto the leader's mbarrier; the leader issues
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16), and each CTA's TMEM
// receives its 128 rows x all 256 columns.  So every SM streams 32 KB per
// 64-deep K step (instead of 48 KB for a one-CTA 128 x 256 tile) for the same
// tensor work, and the MMA's N is always full.
//
// An expert's last pair tile, when it covers only one 128-row M tile (its
// kept rows end in the first half of the 256), is a half tile: each CTA
// loads 64 of the rows (a 64-row box) and the leader issues the M = 128 form
// of tcgen05.mma.cta_group::2, so the tile costs half a pair tile instead of
// padding the expert to 256 rows.  Its accumulator is laid out across the
// pair's TMEM in the 2 x 2 datapath form: in each CTA, TMEM lanes 0-63 hold
// that CTA's 64 rows x output columns 0-127, lanes 64-127 the same rows x
// columns 128-255, both at accumulator columns 0-127.
//
// The epilogue is the one-CTA kernel's (epilogue_rows: one TMEM lane = one
// output row per thread; ReLU and 32 x 32 TMA box stores for the hidden
// activations), run by each CTA on its 128 rows (on a half tile: warps of
// lane quarters 0-1 on the first 128 columns of its 64 rows, quarters 2-3 on
// the last 128).  Two TMEM accumulators
// alternate between tiles; the four epilogue warps of both CTAs hand an
// accumulator back to the leader.  No copy here is multicast.
#include <cstring>

#include "gemm_pair.cuh"

namespace smoe {

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    expert_gemm_pair_rows_kernel(const __grid_constant__ CUtensorMap tmap_a,
                                 const __grid_constant__ CUtensorMap tmap_a64,
                                 const __grid_constant__ CUtensorMap tmap_w,
                                 const __grid_constant__ CUtensorMap tmap_out, GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* stage_out = smem + kPairStages * kPairStageBytes;          // [4][4 KB], 1024-aligned
  uint8_t* tail = stage_out + 4 * kStageOutBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(tail);   // leader: TMA bytes of both CTAs
  uint64_t* empty = full + kPairStages;                  // local: stage free (MMA done)
  uint64_t* tfull = empty + kPairStages;                 // local: accumulator ready
  uint64_t* tempty = tfull + 2;                          // leader: accumulator drained
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tail + 192);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tail + 196);
  int* tok_s = reinterpret_cast<int*>(tail + 256);                      // [4][32]
  int* mts = reinterpret_cast<int*>(tail + 768);                        // [N + 1]
  int* pts = mts + (p.N + 1);                                           // [N + 1]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cid = static_cast<int>(cluster_id_x());
  const int ncl = static_cast<int>(cluster_count_x());
  const long long lim = p.spin;
  const int kblocks = p.K / kBK;

  for (int i = threadIdx.x; i <= p.N; i += blockDim.x) mts[i] = p.mtile_start[i];
  __syncthreads();
  if (warp == 0) pair_prefix_warp(p.N, mts, pts);       // 256-row tiles per expert
  __syncthreads();
  const int total = pts[p.N] * p.ntiles_n;
  if (cid >= total) return;                 // same decision in both CTAs of the pair

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 8);               // 4 epilogue warps x 2 CTAs
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();                          // the peer's barriers exist before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const uint32_t full_lead = map_to_rank(smem_u32(full), 0);
  const uint32_t tempty_lead = map_to_rank(smem_u32(tempty), 0);

  if (warp == 0) {
    // ------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmap_a);
      tma_prefetch_desc(&tmap_a64);
      tma_prefetch_desc(&tmap_w);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_phase = 0;
      bool ok = true;
      for (int tile = cid; tile < total && ok; tile += ncl) {
        if (*abort_flag) break;
        int e, tt, n;
        decode_tile(tile, pts, p.N, p.ntiles_n, e, tt, n);
        const bool half = 2 * tt + 1 == mts[e + 1] - mts[e];   // one 128-row M tile
        const int a_row = static_cast<int>(static_cast<int64_t>(e) * p.C + tt * 256 +
                                           static_cast<int>(rank) * (half ? 64 : 128));
        const int w_row = e * p.n_out + n * kBN + static_cast<int>(rank) * 128;
        const uint32_t tx = 2 * (half ? kPairTokBytes / 2 + kPairWBytes : kPairStageBytes);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, lim)) {
            report_error(p.err, SWITCH_ERR_TIMEOUT, kWhereGemmProducer, tile);
            *abort_flag = 1;
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * kPairStageBytes;
          const uint32_t bar = full_lead + 8u * stage;
          if (leader) mbar_arrive_expect_tx(&full[stage], tx);
          tma_load_2d_pair(sa, half ? &tmap_a64 : &tmap_a, bar, kb * kBK, a_row);
          tma_load_2d_pair(sa + kPairTokBytes, &tmap_w, bar, kb * kBK, w_row);
          issued_mask |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == kPairStages) { stage = 0; phase ^= 1u; }
        }
      }
      // Both CTAs' bytes land on the leader's barriers: the leader waits for
      // every issued stage before the final cluster barrier.
      if (leader) {
        for (int s = 0; s < kPairStages; ++s)
          if (((issued_mask >> s) & 1u) &&
              !mbar_wait_cluster(&full[s], (issued_phase >> s) & 1u, kDefaultSpinCycles))
            report_error(p.err, SWITCH_ERR_TIMEOUT, kWhereDrain, s);
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------- MMA issuer
    if (leader && lane == 0) {
      constexpr uint32_t idesc_full = idesc_bf16_f32(2 * kBM, kBN);
      constexpr uint32_t idesc_half = idesc_bf16_f32(kBM, kBN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool any = false;
      for (int tile = cid; tile < total && !*abort_flag; tile += ncl) {
        int e, tt, n;
        decode_tile(tile, pts, p.N, p.ntiles_n, e, tt, n);
        const uint32_t idesc = 2 * tt + 1 == mts[e + 1] - mts[e] ? idesc_half : idesc_full;
        if (!mbar_wait_cluster(&tempty[acc], acc_phase ^ 1u, lim)) {
          report_error(p.err, SWITCH_ERR_TIMEOUT, kWhereGemmMma, tile);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kBN);
        bool ok = true;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait_cluster(&full[stage], phase, lim)) {
            report_error(p.err, SWITCH_ERR_TIMEOUT, kWhereGemmMma, tile);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * kPairStageBytes);
          const uint32_t sw = sa + kPairTokBytes;
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)
            umma_bf16_pair(d_tmem, sw128_kmajor_desc(sa + k * 32), sw128_kmajor_desc(sw + k * 32),
                           idesc, (kb | k) != 0 ? 1u : 0u);
          any = true;
          umma_commit_pair(&empty[stage], 0x3);
          if (++stage == kPairStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit_pair(&tfull[acc], 0x3);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (any && *abort_flag) {
        umma_commit_pair(drain, 0x1);
        if (!mbar_wait(drain, 0, kDefaultSpinCycles))
          report_error(p.err, SWITCH_ERR_TIMEOUT, kWhereDrain, -1);
      }
    }
  } else if (warp >= 2 && warp < 6) {
    // ------------------------------------------------------- epilogue warps
    const int q = warp & 3;                 // TMEM lane quarter of this warp
    const uint32_t stg = smem_u32(stage_out + q * kStageOutBytes);
    int* tokw = tok_s + q * 32;
    int acc = 0;
    uint32_t acc_phase = 0;
    if (lane == 0 && p.mode != kModeCombine) tma_prefetch_desc(&tmap_out);
    for (int tile = cid; tile < total; tile += ncl) {
      // warp-uniform outcome: the TMEM loads below are warp-collective
      const bool ok = __all_sync(0xffffffffu, mbar_wait_sleepy(&tfull[acc], acc_phase, lim));
      if (!ok) {
        if (lane == 0) {
          report_error(p.err, SWITCH_ERR_TIMEOUT, kWhereGemmEpilogue, tile);
          *abort_flag = 1;
        }
        break;
      }
      tc_fence_after();
      int e, tt, n;
      decode_tile(tile, pts, p.N, p.ntiles_n, e, tt, n);
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc * kBN);
      if (2 * tt + 1 != mts[e + 1] - mts[e]) {
        // this CTA's rows are the 128-row tile 2 tt + rank of the expert
        epilogue_tile(p, &tmap_out, e, 2 * tt + static_cast<int>(rank), n, taddr, stg, tokw, q,
                      lane);
      } else {
        // half tile: rows tt*256 + 64 rank + 32 (q % 2) .., columns
        // n*256 + 128 (q / 2) .., at accumulator columns 0-127
        const int col_base = n * kBN + (q >> 1) * 128;
        const int ncols = p.n_out - col_base < 128 ? p.n_out - col_base : 128;
        if (ncols > 0)
          epilogue_rows(p, &tmap_out, e,
                        static_cast<int64_t>(tt) * 256 + static_cast<int>(rank) * 64 +
                            (q & 1) * 32,
                        col_base, ncols, taddr, stg, tokw, lane);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader) mbar_arrive(&tempty[acc]);
        else mbar_arrive_remote(tempty_lead + 8u * acc);
      }
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    if (lane == 0) bulk_wait_all();        // boxes stored from shared memory are written
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();                          // no CTA leaves while its peer may still signal it
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, kTmemCols);
}

cudaError_t run_gemm_pair_rows(const CUtensorMap& ta, const CUtensorMap& ta64,
                               const CUtensorMap& tw, const CUtensorMap& to,
                               const GemmParams& gp, int num_sms, cudaStream_t st) {
  const size_t smem = gemm_pair_smem_bytes(gp.N);
  static size_t smem_set[64] = {};
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(&expert_gemm_pair_rows_kernel),
                                    smem, smem_set);
  if (e != cudaSuccess) return e;
  const int grid = (num_sms / 2) * 2;
  expert_gemm_pair_rows_kernel<<<grid, kGemmThreads, smem, st>>>(ta, ta64, tw, to, gp);
  return cudaGetLastError();
}

}  // namespace smoe
