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

#include "gemm_common.cuh"

namespace smoe {

constexpr int kPairStages = 6;
constexpr uint32_t kPairWBytes = 128 * kBK * 2;                // 16 KB: 128 weight rows
constexpr uint32_t kPairTokBytes = 128 * kBK * 2;              // 16 KB: up to 128 token rows
constexpr uint32_t kPairStageBytes = kPairWBytes + kPairTokBytes;
constexpr uint32_t kPairTail = 4 * kStageOutBytes + 768;       // + mts, pts

// Prefix over experts of ceil(M tiles / 2) = ceil(rows / 256), one warp.
__device__ void pair_prefix_warp(int N, const int* mts, int* pts) {
  const int lane = threadIdx.x & 31;
  const int per = (N + 31) / 32;
  int s = 0;
  for (int i = 0; i < per; ++i) {
    const int e = lane * per + i;
    if (e < N) s += (mts[e + 1] - mts[e] + 1) >> 1;
  }
  int inc = s;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, inc, off);
    if (lane >= off) inc += v;
  }
  int run = inc - s;
  for (int i = 0; i < per; ++i) {
    const int e = lane * per + i;
    if (e < N) {
      pts[e] = run;
      run += (mts[e + 1] - mts[e] + 1) >> 1;
    }
  }
  if (lane == 31) pts[N] = inc;
}

// Geometry of one pair tile.
struct PairTile {
  int e;        // expert
  int t0;       // first token slot of the tile within the expert
  int nv;       // token slots of the tile that hold a kept token (1..256)
  int nmma;     // MMA N: nv rounded up to 16
  int f0;       // first output feature of the pair tile
};

// Tile order: an expert's token tiles vary fastest, then its feature tiles,
// so clusters running side by side share the weight tile.
__device__ __forceinline__ PairTile pair_tile(const GemmParams& p, const int* pts, int tile) {
  PairTile t;
  int tt, mf;
  decode_tile(tile, pts, p.N, p.ntiles_n, t.e, tt, mf);
  t.t0 = tt * 256;
  const int64_t rem = kept_rows(p, t.e) - t.t0;
  t.nv = rem < 256 ? static_cast<int>(rem) : 256;
  t.nmma = (t.nv + 15) & ~15;
  t.f0 = mf * 256;
  return t;
}

// Two bf16 (the halves of v) to two shared addresses.
__device__ __forceinline__ void st_shared_b16x2(uint32_t a_lo, uint32_t a_hi, uint32_t v) {
  asm volatile(
      "{\n .reg .b16 lo, hi;\n mov.b32 {lo, hi}, %2;\n"
      " st.shared.b16 [%0], lo;\n st.shared.b16 [%1], hi;\n}\n" ::"r"(a_lo),
      "r"(a_hi), "r"(v)
      : "memory");
}

// Combine: per lane, the token id and gate of column c * 32 + lane of a
// tile (c < 8; -1 / 0 past the kept tokens), and the 64-byte residual
// segments of the warp's features pulled into L2 ahead of their reads.
struct CombineMeta {
  int tok[8];
  float g[8];
};

__device__ __forceinline__ void combine_meta(const GemmParams& p, const PairTile& t, int fb,
                                             CombineMeta& m, int lane) {
  const int64_t row0 = static_cast<int64_t>(t.e) * p.C + t.t0;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const int col = c * 32 + lane;
    m.tok[c] = col < t.nv ? p.slot_token[row0 + col] : -1;
  }
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    m.g[c] = 0.f;
    if (m.tok[c] >= 0) {
      m.g[c] = p.gate[m.tok[c]];
      if (p.x_res != nullptr && fb < p.n_out)
        prefetch_l2(p.x_res + static_cast<int64_t>(m.tok[c]) * p.n_out + fb);
    }
  }
}

template <typename V>
__device__ __forceinline__ V pick8(const V (&a)[8], int c) {
  V r = a[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) r = c == i ? a[i] : r;
  return r;
}

// Epilogue of one tile for the calling warp: features fb .. fb + 31 (one per
// lane) of the tile's tokens.  `taddr` addresses this warp's TMEM lanes at
// column 0 of the accumulator; `stg` is the warp's 4 KB shared buffer.
// Hidden / Y: `nbox` counts the boxes this warp has stored (the two 2 KB
// halves of `stg` alternate strictly across tiles).  Combine: `m` holds the
// tile's token ids and gates; a chunk's fp32 values are transposed through
// `stg` so that each lane then owns 8 features of one token and every
// global access moves 16 bytes (8 token rows x 64 bytes per instruction).
__device__ __forceinline__ void epilogue_tile_t(const GemmParams& p, const CUtensorMap* tmap_out,
                                                const PairTile& t, int fb, uint32_t taddr,
                                                uint32_t stg, const CombineMeta& m, int lane,
                                                int& nbox) {
  if (fb >= p.n_out) return;                       // warp-uniform: past the last feature
  const int nch = (t.nv + 31) >> 5;
  const int64_t row0 = static_cast<int64_t>(t.e) * p.C + t.t0;   // slot of token column 0
  const int f = fb + lane;
  // byte offset of this lane's feature inside a 64-byte box row, before the
  // row's swizzle: 16-byte chunk lane / 8, 2-byte element lane % 8
  const uint32_t chunk = static_cast<uint32_t>(lane >> 3);
  const uint32_t within = static_cast<uint32_t>(lane & 7) * 2u;
  const int qq = lane & 3;          // combine: 8-feature group of this lane
  const int rr0 = lane >> 2;        // combine: token row within an 8-row pass

  auto chunk_store = [&](int c, const uint32_t* u) {
    const int j0 = c * 32;
    const int jn = t.nv - j0 < 32 ? t.nv - j0 : 32;     // kept tokens in this chunk
    if (p.mode == kModeCombine) {
      // transpose: element (token j, feature lane) at row j, 16-byte chunk
      // (lane / 4) ^ (j % 8) of a 128-byte row
#pragma unroll
      for (int j = 0; j < 32; ++j)
        st_shared_f32(stg + j * 128 + ((((lane >> 2) ^ j) & 7) << 4) + (lane & 3) * 4,
                      __uint_as_float(u[j]));
      __syncwarp();
      const int tkc = pick8(m.tok, c);
      const float gcl = pick8(m.g, c);
      int tk[4];
      float g[4];
      uint4 xr[4];
#pragma unroll
      for (int pass = 0; pass < 4; ++pass) {
        const int rr = pass * 8 + rr0;
        tk[pass] = __shfl_sync(0xffffffffu, tkc, rr);
        g[pass] = __shfl_sync(0xffffffffu, gcl, rr);
        xr[pass] = make_uint4(0, 0, 0, 0);
        if (tk[pass] >= 0 && p.x_res != nullptr)
          xr[pass] = __ldg(reinterpret_cast<const uint4*>(
              p.x_res + static_cast<int64_t>(tk[pass]) * p.n_out + fb + qq * 8));
      }
#pragma unroll
      for (int pass = 0; pass < 4; ++pass) {
        const int rr = pass * 8 + rr0;
        if (tk[pass] < 0) continue;
        const float4 a = ld_shared_v4(stg + rr * 128 + (((2 * qq) ^ (rr & 7)) << 4));
        const float4 b = ld_shared_v4(stg + rr * 128 + (((2 * qq + 1) ^ (rr & 7)) << 4));
        const float gg = g[pass];
        uint4 o;
        o.x = pack_bf16x2(fmaf(gg, a.x, bf16_lo(xr[pass].x)), fmaf(gg, a.y, bf16_hi(xr[pass].x)));
        o.y = pack_bf16x2(fmaf(gg, a.z, bf16_lo(xr[pass].y)), fmaf(gg, a.w, bf16_hi(xr[pass].y)));
        o.z = pack_bf16x2(fmaf(gg, b.x, bf16_lo(xr[pass].z)), fmaf(gg, b.y, bf16_hi(xr[pass].z)));
        o.w = pack_bf16x2(fmaf(gg, b.z, bf16_lo(xr[pass].w)), fmaf(gg, b.w, bf16_hi(xr[pass].w)));
        *reinterpret_cast<uint4*>(p.comb_out + static_cast<int64_t>(tk[pass]) * p.n_out + fb +
                                  qq * 8) = o;
      }
      __syncwarp();                    // the buffer is rewritten by the next chunk
      return;
    }
    float v[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float a = __uint_as_float(u[j]);
      v[j] = p.mode == kModeHidden ? fmaxf(a, 0.f) : a;
    }
    // Whole 32-row boxes by TMA: in the hidden buffer (internal scratch) any
    // box inside this expert's slots; in Y (the caller's) only kept rows.
    if (p.mode == kModeHidden ? t.t0 + j0 + 32 <= p.C : jn == 32) {
      // transpose through shared memory, one TMA store
      const uint32_t buf = stg + static_cast<uint32_t>(nbox & 1) * 2048u;
      if (lane == 0) bulk_wait_read<1>();          // the box stored from `buf` before is out
      __syncwarp();
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        const uint32_t a0 = buf + j * 64 + ((chunk ^ ((j >> 1) & 3u)) << 4) + within;
        const uint32_t a1 = buf + (j + 1) * 64 + ((chunk ^ (((j + 1) >> 1) & 3u)) << 4) + within;
        st_shared_b16x2(a0, a1, pack_bf16x2(v[j], v[j + 1]));
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(tmap_out, buf, fb, static_cast<int>(row0 + j0));
        bulk_commit();
      }
      ++nbox;
    } else {
      // kept rows only, one 64-byte row segment per store instruction
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (j < jn) p.out[(row0 + j0 + j) * p.ldo + f] = __float2bfloat16_rn(v[j]);
    }
  };

  // Chunk c + 1 is loaded from TMEM while chunk c is stored.
  uint32_t ra[32], rb[32];
  tmem_ld32_issue(taddr, ra);
#pragma unroll 1
  for (int c = 0; c < nch; c += 2) {
    tmem_ld_wait(ra);
    if (c + 1 < nch) tmem_ld32_issue(taddr + static_cast<uint32_t>((c + 1) * 32), rb);
    chunk_store(c, ra);
    if (c + 1 >= nch) break;
    tmem_ld_wait(rb);
    if (c + 2 < nch) tmem_ld32_issue(taddr + static_cast<uint32_t>((c + 2) * 32), ra);
    chunk_store(c + 1, rb);
  }
}

template <bool kGather>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    expert_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_tok,
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
      if (lead_warp && lane == 0 && !kGather) tma_prefetch_desc(&tmap_tok);
      if (lead_warp && lane == 0) tma_prefetch_desc(&tmap_w);
      const int ch = lane & 7;
      const int gw = lead_warp ? 0 : warp - 5;                // 0..3
      const int row0 = 32 * gw + (lane >> 3);                  // rows row0 + 4 j, j < 8
      const uint32_t vec_per_row = static_cast<uint32_t>(p.K / 8);
      const uint32_t sw_even = static_cast<uint32_t>((ch ^ (row0 & 7)) << 4);
      const uint32_t sw_odd = static_cast<uint32_t>((ch ^ ((row0 + 4) & 7)) << 4);
      const uint32_t tx_bytes = kGather ? 2 * kPairWBytes : 2 * kPairStageBytes;
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
            if (!kGather) tma_load_2d_pair(stok, &tmap_tok, bar, kb * kBK, tok_row);
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
    if (lane == 0 && p.mode != kModeCombine) tma_prefetch_desc(&tmap_out);
    if (p.mode == kModeCombine) {
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
      if (p.mode == kModeCombine && tile + ncl < total) {
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
cudaError_t run_gemm_pair(const CUtensorMap& ttok, const CUtensorMap& tw, const CUtensorMap& to,
                          const GemmParams& gp, int num_sms, cudaStream_t st) {
  const size_t smem = gemm_pair_smem_bytes(gp.N);
  static size_t smem_set[64] = {};
  cudaError_t e = ensure_smem_limit(
      reinterpret_cast<const void*>(&expert_gemm_pair_kernel<kGather>), smem, smem_set);
  if (e != cudaSuccess) return e;
  const int grid = (num_sms / 2) * 2;
  expert_gemm_pair_kernel<kGather><<<grid, kGemmThreads, smem, st>>>(ttok, tw, to, gp);
  return cudaGetLastError();
}

template cudaError_t run_gemm_pair<true>(const CUtensorMap&, const CUtensorMap&,
                                         const CUtensorMap&, const GemmParams&, int,
                                         cudaStream_t);
template cudaError_t run_gemm_pair<false>(const CUtensorMap&, const CUtensorMap&,
                                          const CUtensorMap&, const GemmParams&, int,
                                          cudaStream_t);

}  // namespace smoe
