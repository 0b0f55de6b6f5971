// Shared pieces of the tcgen05 grouped expert GEMMs (one-SM and CTA-pair
// kernels): tile geometry, parameters, the device-side tile list, and the
// epilogue that drains one 128-row x 256-column accumulator to memory.
#pragma once

#include "kernels.cuh"

namespace smoe {

// ------------------------------------------------------------- tile list

// Tile t belongs to the expert e with mts[e] * ntn <= t < mts[e + 1] * ntn
// (the last such e, which is never empty).  Inside an expert, M tiles vary
// fastest so that CTAs running side by side share the weight tile.
__device__ __forceinline__ void decode_tile(int tile, const int* mts, int N, int ntn, int& e,
                                            int& m, int& n) {
  int lo = 0, hi = N;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (mts[mid] * ntn <= tile) lo = mid; else hi = mid;
  }
  e = lo;
  const int mt = mts[e + 1] - mts[e];
  const int local = tile - mts[e] * ntn;
  n = local / mt;
  m = local - n * mt;
}

constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr uint32_t kABytes = kBM * kBK * 2;             // 16 KB
constexpr uint32_t kBBytes = kBN * kBK * 2;             // 32 KB
// w0 producer (weights + A rows 0-31), w1 MMA, w2-5 epilogue, w6-8 producers
// (A rows 32-127 when rows are gathered)
constexpr int kGemmThreads = 288;
constexpr int kGatherWarps = 4;
constexpr int kGatherLanes = 32 * kGatherWarps;
constexpr uint32_t kTmemCols = 512;                     // 2 accumulators x 256
constexpr uint32_t kStageOutBytes = 32 * 32 * 4;        // per epilogue warp: 32 rows x 32 fp32
constexpr uint32_t kTailBytes = 4 * kStageOutBytes + 128 + 4 * 32 * 4;   // + mts[N + 1]

struct GemmParams {
  int N, n_out, K, ntiles_n;
  int64_t C;
  const int* counts;
  const int* mtile_start;
  const int* slot_token;
  const __nv_bfloat16* a_rows;  // gather mode: x [T, K]
  int mode;
  __nv_bfloat16* out;       // kModeHidden / kModeY: row e*C + r, leading dim ldo
  int64_t ldo;
  const __nv_bfloat16* x_res;   // kModeCombine
  const float* gate;
  __nv_bfloat16* comb_out;      // [T, n_out]
  __nv_bfloat16* peer_out[kEpMaxRanks];   // kModeCombineEp: each rank's output rows
  DevErr* err;
  long long spin;
  // kModeCombine on CTA pairs: x_res is the dispatched buffer and a slot's
  // residual row is its own row there (a copy of x[token]), so a tile reads
  // consecutive rows instead of its tokens' scattered rows of x.
  bool res_by_slot;
  // CTA-pair kernel: take the tile list from its end (the last experts
  // first).  Right after GEMM1 the last experts' hidden rows are the ones
  // still in L2, so GEMM2 reads them before they are evicted.
  bool reverse_tiles;
};

// Rows (m*128 + r) of expert e in this tile that hold a token.
__device__ __forceinline__ int64_t kept_rows(const GemmParams& p, int e) {
  const int64_t cnt = p.counts[e];
  return cnt < p.C ? cnt : p.C;
}


// Combine epilogue: the token whose row this thread drains in a given tile
// (row m * 128 + q * 32 + lane of expert e), or -1.
__device__ __forceinline__ int combine_row_token(const GemmParams& p, int e, int m, int q,
                                                 int lane) {
  const int64_t r = static_cast<int64_t>(m) * kBM + q * 32 + lane;
  return r < kept_rows(p, e) ? p.slot_token[static_cast<int64_t>(e) * p.C + r] : -1;
}

// Pull a token's residual row segment (256 columns of x) into L2 ahead of
// the tile that adds it, so the epilogue's reads do not wait on DRAM.
__device__ __forceinline__ void prefetch_residual(const GemmParams& p, int tok, int n) {
  if (tok < 0 || p.x_res == nullptr) return;
  const char* base = reinterpret_cast<const char*>(p.x_res + static_cast<int64_t>(tok) * p.n_out +
                                                   n * kBN);
  const int bytes = (p.n_out - n * kBN < kBN ? p.n_out - n * kBN : kBN) * 2;
  for (int off = 0; off < bytes; off += 128) prefetch_l2(base + off);
}

// Epilogue of one tile for the calling warp (quarter q of the accumulator's
// 128 TMEM lanes: rows m * 128 + q * 32 + lane of expert e).  Each thread
// owns one accumulator row.  The 32-column chunks are read from TMEM one
// ahead of their use, so a chunk's load is in flight while the previous one
// is stored.  Two store paths, both through the warp's 4 KB shared buffer
// `stg` (1024-byte aligned):
//   * hidden / Y rows, when all 32 rows of the quarter hold tokens: ReLU (or
//     nothing) + bf16 into a 32 x 32 box in the 64-byte-swizzled layout,
//     written out by one TMA store per chunk (two boxes alternate);
//   * otherwise (combine, or a quarter with padding rows): fp32 values are
//     transposed through the buffer so that each global store instruction
//     writes 8 rows x 64 bytes, rows past the expert's count skipped; the
//     combine adds the residual row and scales by the token's gate.
// The general form: the warp's 32 rows start at row `rbase` of expert e,
// and its accumulator holds `ncols` output columns from `col_base` (a
// multiple of 64) on, read from TMEM at taddr, taddr + 32, ...
__device__ __forceinline__ void epilogue_rows(const GemmParams& p, const CUtensorMap* tmap_out,
                                              int e, int64_t rbase, int col_base, int ncols,
                                              uint32_t taddr, uint32_t stg, int* tokw,
                                              int lane) {
  const int qq = lane & 3;          // 8-column group in the transposed pass
  const int rr0 = lane >> 2;        // row within an 8-row pass
  const int64_t n_e = kept_rows(p, e);
  const bool valid = rbase + lane < n_e;
  const bool bulk = p.mode != kModeCombine && rbase + 32 <= n_e;
  const int nch = ncols / 32;       // even: n_out % 64 == 0
  float g = 1.f;
  if (p.mode == kModeCombine) {
    const int tk = valid ? p.slot_token[static_cast<int64_t>(e) * p.C + rbase + lane] : 0;
    g = valid ? p.gate[tk] : 0.f;
    tokw[lane] = tk;
  }
  if (!bulk && p.mode != kModeCombine) {
    if (lane == 0) bulk_wait_read<0>();      // earlier boxes have left the buffer
  }
  __syncwarp();
  const int box_row = static_cast<int>(static_cast<int64_t>(e) * p.C + rbase);
  const uint32_t swz = static_cast<uint32_t>((lane >> 1) & 3);

  auto chunk_bulk = [&](int c, const uint32_t* v) {
    uint32_t pk[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      float a = __uint_as_float(v[2 * j]), b = __uint_as_float(v[2 * j + 1]);
      if (p.mode == kModeHidden) { a = fmaxf(a, 0.f); b = fmaxf(b, 0.f); }
      pk[j] = pack_bf16x2(a, b);
    }
    const uint32_t buf = stg + static_cast<uint32_t>(c & 1) * 2048u;
    if (lane == 0) bulk_wait_read<1>();      // the box stored from `buf` two chunks ago is out
    __syncwarp();
#pragma unroll
    for (int k = 0; k < 4; ++k)
      st_shared_v4u(buf + lane * 64 + ((static_cast<uint32_t>(k) ^ swz) << 4), pk[4 * k],
                    pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(tmap_out, buf, col_base + c * 32, box_row);
      bulk_commit();
    }
  };

  auto chunk_lsu = [&](int c, const uint32_t* u) {
    const int col0 = col_base + c * 32;
    float v[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float a = __uint_as_float(u[j]);
      v[j] = p.mode == kModeHidden ? fmaxf(a, 0.f) : (p.mode == kModeCombine ? g * a : a);
    }
#pragma unroll
    for (int k = 0; k < 8; ++k)
      st_shared_v4(stg + lane * 128 + ((k ^ (lane & 7)) << 4), v[4 * k], v[4 * k + 1],
                   v[4 * k + 2], v[4 * k + 3]);
    __syncwarp();
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) {
      const int rr = pass * 8 + rr0;
      const int64_t r = rbase + rr;
      if (r < n_e) {
        const float4 a = ld_shared_v4(stg + rr * 128 + (((2 * qq) ^ (rr & 7)) << 4));
        const float4 b = ld_shared_v4(stg + rr * 128 + (((2 * qq + 1) ^ (rr & 7)) << 4));
        uint4 o;
        if (p.mode == kModeCombine) {
          const int tk = tokw[rr];
          const int64_t off = static_cast<int64_t>(tk) * p.n_out + col0 + qq * 8;
          uint4 xr = make_uint4(0, 0, 0, 0);
          if (p.x_res != nullptr) xr = __ldg(reinterpret_cast<const uint4*>(p.x_res + off));
          o.x = pack_bf16x2(a.x + bf16_lo(xr.x), a.y + bf16_hi(xr.x));
          o.y = pack_bf16x2(a.z + bf16_lo(xr.y), a.w + bf16_hi(xr.y));
          o.z = pack_bf16x2(b.x + bf16_lo(xr.z), b.y + bf16_hi(xr.z));
          o.w = pack_bf16x2(b.z + bf16_lo(xr.w), b.w + bf16_hi(xr.w));
          *reinterpret_cast<uint4*>(p.comb_out + off) = o;
        } else {
          o.x = pack_bf16x2(a.x, a.y);
          o.y = pack_bf16x2(a.z, a.w);
          o.z = pack_bf16x2(b.x, b.y);
          o.w = pack_bf16x2(b.z, b.w);
          *reinterpret_cast<uint4*>(p.out + (static_cast<int64_t>(e) * p.C + r) * p.ldo +
                                    col0 + qq * 8) = o;
        }
      }
    }
    __syncwarp();
  };

  // Chunk c + 1 is loaded while chunk c is stored (nch is even).
  uint32_t ra[32], rb[32];
  tmem_ld32_issue(taddr, ra);
#pragma unroll 1
  for (int c = 0; c < nch; c += 2) {
    tmem_ld_wait(ra);
    tmem_ld32_issue(taddr + static_cast<uint32_t>((c + 1) * 32), rb);
    if (bulk) chunk_bulk(c, ra); else chunk_lsu(c, ra);
    tmem_ld_wait(rb);
    if (c + 2 < nch) tmem_ld32_issue(taddr + static_cast<uint32_t>((c + 2) * 32), ra);
    if (bulk) chunk_bulk(c + 1, rb); else chunk_lsu(c + 1, rb);
  }
}

// One 128-row x 256-column tile (M tile m, column tile n): warp q drains rows
// m * 128 + q * 32 .. + 31, all the tile's columns.
__device__ __forceinline__ void epilogue_tile(const GemmParams& p, const CUtensorMap* tmap_out,
                                              int e, int m, int n, uint32_t taddr, uint32_t stg,
                                              int* tokw, int q, int lane) {
  epilogue_rows(p, tmap_out, e, static_cast<int64_t>(m) * kBM + q * 32, n * kBN,
                p.n_out - n * kBN < kBN ? p.n_out - n * kBN : kBN, taddr, stg, tokw, lane);
}

// Row-major CTA-pair kernel launcher (expert_ffn_pair_rows.cu): 256-row x
// 256-column tiles of row-contiguous operands (no gather).
cudaError_t run_gemm_pair_rows(const CUtensorMap& ta, const CUtensorMap& ta64,
                               const CUtensorMap& tw, const CUtensorMap& to,
                               const GemmParams& gp, int num_sms, cudaStream_t st);
// Dynamic shared memory of the CTA-pair kernels for N experts.
size_t gemm_pair_smem_bytes(int N);

// CTA-pair kernel launcher (expert_ffn_pair.cu).  ta, ta64, ta32: the token
// rows with 128-, 64- and 32-row boxes (unused when gathered).
template <bool kGather>
cudaError_t run_gemm_pair(const CUtensorMap& ta, const CUtensorMap& ta64, const CUtensorMap& ta32,
                          const CUtensorMap& tb, const CUtensorMap& to, const GemmParams& gp,
                          int num_sms, cudaStream_t st);

}  // namespace smoe
