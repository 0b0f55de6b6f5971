// Expert FFN GEMMs on CTA pairs (2-SM tcgen05) with the operands swapped:
// the accumulator holds the transposed tile, output features x tokens,
//
//   D[f, j] = sum_k W[e][f, k] * A[token j, k]      (W: w1 [F, d] or w2 [d, F]).
//
// A pair tile is 256 output features x up to 256 of one expert's tokens.  An
// expert's last token tile is ragged; the MMA's N is set to its token count
// rounded up to 16, so an expert wastes at most 15 token columns instead of
// padding its rows to a whole 128- or 256-row M tile.
//
//   * CTA r of the pair holds weight rows f0 + 128 r .. + 127 (the A operand,
//     by TMA) and token rows r * N/2 .. (r + 1) * N/2 - 1 of the tile (the B
//     operand: gathered from x through slot_token with 16-byte cp.async in
//     GEMM1, or by TMA from a row-contiguous buffer).  The leader (r = 0)
//     issues tcgen05.mma.cta_group::2 (M = 256, N = 16..256, K = 16); each
//     CTA's TMEM receives its 128 features x N tokens.  Every SM streams 32 KB
//     per 64-deep K step; the ring is six stages deep.
//   * Weight (and tiled token) copies are TMA loads whose byte counts land on
//     the leader's mbarrier; gathered rows are signalled on a local barrier
//     and relayed to the leader by the follower.
//   * Commits are multicast to both CTAs (stage release, accumulator ready);
//     both CTAs' epilogue warps hand an accumulator back to the leader.
//   * Epilogue (one warp per 32 features): per 32-token chunk a thread owns
//     one feature of 32 tokens.  Hidden / Y: ReLU (or not) + bf16, written
//     transposed into a [32 tokens x 32 features] shared box (64-byte
//     swizzle) and stored by TMA into the token-major buffer.  Combine: the
//     fp32 chunk is transposed through shared memory, then each lane adds
//     gate * acc to 8 features of one token's residual row, 16 bytes per
//     access (out = x + gate * acc, one rounding).
// No copy here is multicast: each CTA loads only its own operands.
#include <cstring>

#include "gemm_pair.cuh"

namespace smoe {

// Token rows per CTA of a tile (nmma / 2) decide its token box when the rows
// come by TMA: 32, 64 or 128 rows, so a ragged tile with few tokens does not
// stream a full 128-row box (its MMA reads only nmma / 2 rows per CTA).
__device__ __forceinline__ int tok_box_rows(int nmma) {
  return nmma <= 64 ? 32 : (nmma <= 128 ? 64 : 128);
}

template <bool kGather>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    expert_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_tok,
                            const __grid_constant__ CUtensorMap tmap_tok64,
                            const __grid_constant__ CUtensorMap tmap_tok32,
                            const __grid_constant__ CUtensorMap tmap_w,
                            const __grid_constant__ CUtensorMap tmap_out, GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* stage_out = smem + kPairStages * kPairStageBytes;          // [4][4 KB], 1024-aligned
  uint8_t* tail = stage_out + 4 * kStageOutBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(tail);   // leader: TMA bytes of both CTAs
  uint64_t* afull = full + kPairStages;                  // local: gathered token rows
  uint64_t* empty = afull + kPairStages;                 // local: stage free (MMA done)
  uint64_t* tfull = empty + kPairStages;                 // local: accumulator ready
  uint64_t* tempty = tfull + 2;                          // leader: accumulator drained
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tail + 192);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tail + 196);
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
  if (warp == 0) pair_prefix_warp(p.N, mts, pts);
  __syncthreads();
  const int total = pts[p.N] * p.ntiles_n;
  if (cid >= total) return;                 // same decision in both CTAs of the pair

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(&full[s], kGather ? 2 : 1);   // leader's expect_tx (+ follower's relay)
      mbar_init(&afull[s], kGatherLanes);
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

  if (warp == 0 || warp >= 6) {
    // ------------------------------------------------------- producer warps
    // warp 0: weights (and tiled token rows) by TMA, plus gathered token rows
    // 0-31; warps 6-8: gathered token rows 32-127.  Gather lane mapping:
    // lane = (row lane / 8 within a group of 4 rows, 16-byte chunk lane % 8),
    // each chunk placed where the 128-byte swizzle puts it (chunk ^ row % 8).
    const bool lead_warp = warp == 0;
    if (!kGather && !lead_warp) goto producer_done;
    {
      if (lead_warp && lane == 0 && !kGather) {
        tma_prefetch_desc(&tmap_tok);
        tma_prefetch_desc(&tmap_tok64);
        tma_prefetch_desc(&tmap_tok32);
      }
      if (lead_warp && lane == 0) tma_prefetch_desc(&tmap_w);
      const int ch = lane & 7;
      const int gw = lead_warp ? 0 : warp - 5;                // 0..3
      const int row0 = 32 * gw + (lane >> 3);                  // rows row0 + 4 j, j < 8
      const uint32_t vec_per_row = static_cast<uint32_t>(p.K / 8);
      const uint32_t sw_even = static_cast<uint32_t>((ch ^ (row0 & 7)) << 4);
      const uint32_t sw_odd = static_cast<uint32_t>((ch ^ ((row0 + 4) & 7)) << 4);
      // bytes the TMA copies of one stage bring (both CTAs): the weights, plus
      // the token rows' box when they come by TMA (gathered rows: cp.async)
      auto tx_bytes_of = [&](const PairTile& t) {
        return kGather ? 2 * kPairWBytes
                       : 2 * (kPairWBytes + static_cast<uint32_t>(tok_box_rows(t.nmma)) * kBK * 2);
      };
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_phase = 0;
      uint32_t roff[8];
      // this CTA's token rows of a tile: 16-byte-unit offsets in x (~0u: none)
      auto load_rows = [&](int t_tile, uint32_t* dst) {
        const PairTile t = pair_tile(p, pts, t_tile);
        const int half = t.nmma >> 1;
        const int base = t.t0 + static_cast<int>(rank) * half;   // first token of this CTA
        const int64_t slot0 = static_cast<int64_t>(t.e) * p.C + base;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int r = row0 + 4 * j;
          dst[j] = (r < half && base + r < t.t0 + t.nv)
                       ? static_cast<uint32_t>(p.slot_token[slot0 + r]) * vec_per_row
                       : ~0u;
        }
      };
      if (kGather) load_rows(cid, roff);
      for (int tile = cid; tile < total; tile += ncl) {
        if (__shfl_sync(0xffffffffu, *abort_flag, 0)) break;   // warp-uniform
        const PairTile t = pair_tile(p, pts, tile);
        const int tok_row = static_cast<int>(static_cast<int64_t>(t.e) * p.C + t.t0 +
                                             static_cast<int>(rank) * (t.nmma >> 1));
        const int w_row = t.e * p.n_out + t.f0 + static_cast<int>(rank) * 128;
        const uint32_t tx_bytes = tx_bytes_of(t);
        const int box_rows = tok_box_rows(t.nmma);
        const CUtensorMap* tmap_t = box_rows == 32 ? &tmap_tok32
                                   : (box_rows == 64 ? &tmap_tok64 : &tmap_tok);
        uint32_t roff_next[8];
        const int next = tile + ncl;
        if (kGather && next < total) load_rows(next, roff_next);   // in flight meanwhile
        bool ok = true;
        for (int kb = 0; kb < kblocks; ++kb) {
          int w_ok = 1;
          if (lane == 0) w_ok = mbar_wait(&empty[stage], phase ^ 1u, lim) ? 1 : 0;
          w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
          if (!w_ok) {
            if (lane == 0) {
              report_error(p.err, SWITCH_ERR_TIMEOUT, kWhereGemmProducer, tile);
              *abort_flag = 1;
            }
            ok = false;
            break;
          }
          uint8_t* sw = smem + stage * kPairStageBytes;
          uint8_t* stok = sw + kPairWBytes;
          if (kGather) {
            const uint4* src0 = reinterpret_cast<const uint4*>(p.a_rows) + kb * 8 + ch;
            const uint32_t dst0 = smem_u32(stok) + static_cast<uint32_t>(row0 * 128);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              if (roff[j] != ~0u)
                cp_async16_s(dst0 + j * 512 + ((j & 1) ? sw_odd : sw_even), src0 + roff[j]);
            }
            cp_async_mbar_arrive_noinc(&afull[stage]);
          }
          if (lead_warp && lane == 0) {
            const uint32_t bar = full_lead + 8u * stage;
            if (leader) mbar_arrive_expect_tx(&full[stage], tx_bytes);
            tma_load_2d_pair(sw, &tmap_w, bar, kb * kBK, w_row);
            if (!kGather) tma_load_2d_pair(stok, tmap_t, bar, kb * kBK, tok_row);
          }
          issued_mask |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == kPairStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if (kGather) {
#pragma unroll
          for (int j = 0; j < 8; ++j) roff[j] = roff_next[j];
        }
      }
      // Never leave with copies in flight into shared memory: own cp.async
      // here; both CTAs' TMA bytes complete on the leader's barriers, which
      // the leader drains before the final cluster barrier.
      if (kGather) cp_async_wait_all();
      if (lead_warp && lane == 0 && leader) {
        for (int s = 0; s < kPairStages; ++s)
          if (((issued_mask >> s) & 1u) &&
              !mbar_wait_cluster(&full[s], (issued_phase >> s) & 1u, kDefaultSpinCycles))
            report_error(p.err, SWITCH_ERR_TIMEOUT, kWhereDrain, s);
      }
    }
  producer_done:;
  } else if (warp == 1) {
    if (leader && lane == 0) {
      // ----------------------------------------------------- MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool any = false;
      for (int tile = cid; tile < total && !*abort_flag; tile += ncl) {
        const uint32_t idesc = idesc_bf16_f32(2 * kBM, pair_tile(p, pts, tile).nmma);
        if (!mbar_wait_cluster(&tempty[acc], acc_phase ^ 1u, lim)) {
          report_error(p.err, SWITCH_ERR_TIMEOUT, kWhereGemmMma, tile);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kBN);
        bool ok = true;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait_cluster(&full[stage], phase, lim) ||
              (kGather && !mbar_wait(&afull[stage], phase, lim))) {
            report_error(p.err, SWITCH_ERR_TIMEOUT, kWhereGemmMma, tile);
            *abort_flag = 1;
            ok = false;
            break;
          }
          if (kGather) fence_proxy_async_smem();   // cp.async data -> tensor-core reads
          tc_fence_after();
          const uint32_t sw = smem_u32(smem + stage * kPairStageBytes);
          const uint32_t stok = sw + kPairWBytes;
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)
            umma_bf16_pair(d_tmem, sw128_kmajor_desc(sw + k * 32),
                           sw128_kmajor_desc(stok + k * 32), idesc, (kb | k) != 0 ? 1u : 0u);
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
    } else if (!leader && lane == 0 && kGather) {
      // ------------------------------------------- follower: relay token rows
      // Tell the leader when this CTA's gathered rows of each stage landed.
      int stage = 0;
      uint32_t phase = 0;
      for (int tile = cid; tile < total && !*abort_flag; tile += ncl) {
        bool ok = true;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&afull[stage], phase, lim)) {
            report_error(p.err, SWITCH_ERR_TIMEOUT, kWhereGemmProducer, tile);
            *abort_flag = 1;
            ok = false;
            break;
          }
          fence_proxy_async_smem();
          mbar_arrive_remote(full_lead + 8u * stage);
          if (++stage == kPairStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
      }
    }
  } else {
    // ------------------------------------------------------- epilogue warps
    const int q = warp & 3;                 // TMEM lane quarter of this warp
    const uint32_t stg = smem_u32(stage_out + q * kStageOutBytes);
    int acc = 0;
    uint32_t acc_phase = 0;
    int nbox = 0;
    // combine: token ids / gates of the next tile, fetched (and its residual
    // segments prefetched) while that tile's main loop runs
    CombineMeta meta;
    const int fq = static_cast<int>(rank) * 128 + q * 32;    // warp's feature offset in a tile
    const bool combine = p.mode == kModeCombine || p.mode == kModeCombineEp;
    if (lane == 0 && !combine) tma_prefetch_desc(&tmap_out);
    if (combine) {
      const PairTile t = pair_tile(p, pts, cid);
      combine_meta(p, t, t.f0 + fq, meta, lane);
    }
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
      const PairTile t = pair_tile(p, pts, tile);
      epilogue_tile_t(p, &tmap_out, t, t.f0 + fq,
                      tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                          static_cast<uint32_t>(acc * kBN),
                      stg, meta, lane, nbox);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader) mbar_arrive(&tempty[acc]);
        else mbar_arrive_remote(tempty_lead + 8u * acc);
      }
      if (combine && tile + ncl < total) {
        const PairTile tn = pair_tile(p, pts, tile + ncl);
        combine_meta(p, tn, tn.f0 + fq, meta, lane);
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

size_t gemm_pair_smem_bytes(int N) {
  return 1024 + kPairStages * kPairStageBytes + kPairTail + 2 * sizeof(int) * (N + 1);
}

template <bool kGather>
cudaError_t run_gemm_pair(const CUtensorMap& ttok, const CUtensorMap& ttok64,
                          const CUtensorMap& ttok32, const CUtensorMap& tw, const CUtensorMap& to,
                          const GemmParams& gp, int num_sms, cudaStream_t st) {
  const size_t smem = gemm_pair_smem_bytes(gp.N);
  static size_t smem_set[64] = {};
  cudaError_t e = ensure_smem_limit(
      reinterpret_cast<const void*>(&expert_gemm_pair_kernel<kGather>), smem, smem_set);
  if (e != cudaSuccess) return e;
  const int grid = (num_sms / 2) * 2;
  expert_gemm_pair_kernel<kGather><<<grid, kGemmThreads, smem, st>>>(ttok, ttok64, ttok32, tw,
                                                                      to, gp);
  return cudaGetLastError();
}

template cudaError_t run_gemm_pair<true>(const CUtensorMap&, const CUtensorMap&,
                                         const CUtensorMap&, const CUtensorMap&,
                                         const CUtensorMap&, const GemmParams&, int,
                                         cudaStream_t);
template cudaError_t run_gemm_pair<false>(const CUtensorMap&, const CUtensorMap&,
                                          const CUtensorMap&, const CUtensorMap&,
                                          const CUtensorMap&, const GemmParams&, int,
                                          cudaStream_t);

}  // namespace smoe
