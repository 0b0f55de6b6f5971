// Pieces of the CTA-pair expert GEMM kernel (expert_ffn_pair.cu): stage
// geometry, the pair-tile list, and the epilogue of a swapped tile (output
// features x tokens).
#pragma once

#include "gemm_common.cuh"

namespace smoe {

constexpr int kPairStages = 6;
constexpr uint32_t kPairWBytes = 128 * kBK * 2;                // 16 KB: 128 weight rows
constexpr uint32_t kPairTokBytes = 128 * kBK * 2;              // 16 KB: up to 128 token rows
constexpr uint32_t kPairStageBytes = kPairWBytes + kPairTokBytes;
constexpr uint32_t kPairTail = 4 * kStageOutBytes + 768;       // + mts, pts

// Prefix over experts of ceil(M tiles / 2) = ceil(rows / 256), one warp.
static __device__ void pair_prefix_warp(int N, const int* mts, int* pts) {
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
  if (p.reverse_tiles) tile = pts[p.N] * p.ntiles_n - 1 - tile;
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

// Expert parallelism (kModeCombineEp): `tok` holds the slot's packed source
// (home rank, token), the gate is the slot's, and the residual is the slot's
// own row of the dispatched buffer (a copy of x[token] on this GPU).
__device__ __forceinline__ void combine_meta(const GemmParams& p, const PairTile& t, int fb,
                                             CombineMeta& m, int lane) {
  const int64_t row0 = static_cast<int64_t>(t.e) * p.C + t.t0;
  const bool ep = p.mode == kModeCombineEp;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const int col = c * 32 + lane;
    m.tok[c] = col < t.nv ? p.slot_token[row0 + col] : -1;
  }
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    m.g[c] = 0.f;
    if (m.tok[c] >= 0) {
      const int64_t res_row =
          (ep || p.res_by_slot) ? row0 + c * 32 + lane : static_cast<int64_t>(m.tok[c]);
      m.g[c] = p.gate[ep ? row0 + c * 32 + lane : m.tok[c]];
      if (p.x_res != nullptr && fb < p.n_out)
        prefetch_l2(p.x_res + res_row * p.n_out + fb);
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
    if (p.mode == kModeCombine || p.mode == kModeCombineEp) {
      const bool ep = p.mode == kModeCombineEp;
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
        const int64_t res_row =
            (ep || p.res_by_slot) ? row0 + j0 + rr : static_cast<int64_t>(tk[pass]);
        if (tk[pass] >= 0 && p.x_res != nullptr)
          xr[pass] = __ldg(reinterpret_cast<const uint4*>(p.x_res + res_row * p.n_out + fb +
                                                          qq * 8));
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
        __nv_bfloat16* orow =
            ep ? p.peer_out[tk[pass] >> kEpRankShift] +
                     static_cast<int64_t>(tk[pass] & ((1 << kEpRankShift) - 1)) * p.n_out
               : p.comb_out + static_cast<int64_t>(tk[pass]) * p.n_out;
        *reinterpret_cast<uint4*>(orow + fb + qq * 8) = o;
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

}  // namespace smoe
