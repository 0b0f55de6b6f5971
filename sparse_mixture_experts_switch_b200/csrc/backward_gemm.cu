// Backward GEMMs of the expert FFNs ("Switch Transformers: scaling to
// trillion-parameter models", section "The Core Idea": N independent ReLU
// FFNs over the tokens of each expert's capacity buffer; gradients by the
// chain rule through E_e(x) = relu(x W1_e^T) W2_e^T scaled by the gate,
// section "Switch Routing: From Top-k to k = 1", combine equation).
//
// One persistent tcgen05 kernel, 128 x 256 tiles, K in blocks of 64 through
// a 4-stage ring (TMA, 128-byte swizzle), two 256-column TMEM accumulators.
// Operands that are stored with M (or N) contiguous are fed as MN-major
// shared-memory tiles (64 x 64 TMA boxes, the MN-major canonical layout),
// so no operand is ever transposed in memory.  Two schedules:
//   * rows: tiles (expert, 128 kept slots, 256 columns) from the device
//     tile table, K fixed -- dH = dY . W2_e and dX = dA . W1_e;
//   * weight: tiles (expert, 128 rows, 256 columns) of an expert's weight
//     gradient, K = the expert's kept slots (ragged, from the device counts;
//     3-D tensor maps read zeros past the capacity) -- dW2_e = dY^T H and
//     dW1_e = dA^T X.
// Epilogues (one TMEM lane = one output row per thread):
//   * dH: dA = dH where H > 0 (the ReLU mask), and the row's partial dot
//     product with H for the gate gradient (sum over the tile's columns);
//   * store: bf16 rows of a weight gradient (zeros for an expert with no
//     tokens);
//   * dX: dx[token] = dout[token] (residual) + router term + dX row;
//   * dX per slot (top-2, where two slots can hold one token): the fp32 row
//     (router term + dX row) stored at the slot, added per token afterwards.
#include <cstring>

#include "gemm_common.cuh"
#include "backward.cuh"

namespace smoe {

namespace {

constexpr int kBwdStages = 4;
constexpr uint32_t kBwdStageBytes = kABytes + kBBytes;   // 48 KB
constexpr int kBwdThreads = 192;                         // w0 TMA, w1 MMA, w2-5 epilogue
constexpr uint32_t kBox = 64 * 64 * 2;                   // one 64 x 64 bf16 box, 8 KB

struct BTile {
  int e, m, n, kblocks;
};

template <int kSched>
__device__ __forceinline__ BTile bwd_tile(const BwdParams& p, const int* mts, int t) {
  BTile r;
  if (kSched == kSchedRows) {
    decode_tile(t, mts, p.N, p.ntiles_n, r.e, r.m, r.n);
    r.kblocks = p.K / kBK + p.kx_terms * p.kx_blocks;
  } else if (kSched == kSchedSplit) {
    const int per = p.ntiles_m * p.ntiles_n;
    r.e = t / per;                       // term * nsplit + chunk
    const int local = t - r.e * per;
    r.n = local / p.ntiles_m;
    r.m = local - r.n * p.ntiles_m;
    const int64_t c0 = static_cast<int64_t>(r.e % p.nsplit) * p.split_len;
    const int64_t rem = p.split_rows - c0;
    const int64_t rows = rem < p.split_len ? rem : p.split_len;
    r.kblocks = rows > 0 ? static_cast<int>((rows + kBK - 1) / kBK) : 0;
  } else {
    const int per = p.ntiles_m * p.ntiles_n;
    r.e = t / per;
    const int local = t - r.e * per;
    r.n = local / p.ntiles_m;
    r.m = local - r.n * p.ntiles_m;
    const int64_t cnt = p.counts[r.e];
    const int64_t ne = cnt < p.C ? cnt : p.C;
    r.kblocks = static_cast<int>((ne + kBK - 1) / kBK);
  }
  return r;
}

__device__ __forceinline__ uint4 ld_u4(const void* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

// ---------------------------------------------------------------- epilogues

// Pull the global rows the epilogue of tile t will read for this thread's
// accumulator row into L2 (H for dH; the token's dout row for dX), so that
// the next tile's epilogue does not wait on DRAM.
template <int kEpi>
__device__ __forceinline__ void prefetch_epilogue_rows(const BwdParams& p, const BTile& t, int q,
                                                       int lane) {
  if (kEpi != kEpiDH && kEpi != kEpiDX) return;
  const int64_t r_in = static_cast<int64_t>(t.m) * kBM + q * 32 + lane;
  const int64_t cnt = p.counts[t.e];
  const int64_t lim = kEpi == kEpiDH ? p.C : (cnt < p.C ? cnt : p.C);
  if (r_in >= lim) return;
  const int64_t s = static_cast<int64_t>(t.e) * p.C + r_in;
  const int cols = p.n_out - t.n * kBN < kBN ? p.n_out - t.n * kBN : kBN;
  const char* base;
  if (kEpi == kEpiDH) {
    base = reinterpret_cast<const char*>(p.h + s * p.n_out + t.n * kBN);
  } else {
    if (!p.residual) return;
    base = reinterpret_cast<const char*>(p.dout + static_cast<int64_t>(p.slot_token[s]) * p.n_out +
                                         t.n * kBN);
  }
  for (int off = 0; off < cols * 2; off += 128) prefetch_l2(base + off);
}

// One 32-row x 32-column bf16 chunk of a warp's rows, stored by TMA: the
// lane's 16 packed words go into the 64-byte-swizzled box `buf` (two boxes
// of a warp alternate; the store that last used this one must have read
// it), then lane 0 issues the box store at (col, row).
__device__ __forceinline__ void store_box(const CUtensorMap* map, uint32_t stg, int& nbox,
                                          const uint32_t* pk, int col, int row, int lane) {
  const uint32_t buf = stg + static_cast<uint32_t>(nbox & 1) * 2048u;
  const uint32_t swz = static_cast<uint32_t>((lane >> 1) & 3);
  if (lane == 0) bulk_wait_read<1>();
  __syncwarp();
#pragma unroll
  for (int k = 0; k < 4; ++k)
    st_shared_v4u(buf + lane * 64 + ((static_cast<uint32_t>(k) ^ swz) << 4), pk[4 * k],
                  pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(map, buf, col, row);
    bulk_commit();
  }
  ++nbox;
}

// Weight gradient rows: out[e * M_out + r, n * 256 + ...] = acc, as bf16
// (or fp32 partial sums with kF32).  bf16 chunks of a warp whose 32 rows
// are all inside the weight go out as TMA box stores.
template <bool kF32>
__device__ __forceinline__ void epi_store(const BwdParams& p, const CUtensorMap* tmap_out,
                                          const BTile& t, uint32_t taddr, int q, int lane,
                                          uint32_t stg, int& nbox) {
  const int r = t.m * kBM + q * 32 + lane;
  const bool rv = r < p.M_out;
  const bool bulk = !kF32 && t.m * kBM + q * 32 + 32 <= p.M_out;
  const int box_row = t.e * p.M_out + t.m * kBM + q * 32;
  const int cols = p.n_out - t.n * kBN < kBN ? p.n_out - t.n * kBN : kBN;
  const int64_t ooff = (static_cast<int64_t>(t.e) * p.M_out + r) * p.n_out + t.n * kBN;
  __nv_bfloat16* orow = p.out + ooff;
  auto process = [&](int c, const uint32_t* v) {
    if (bulk) {
      uint32_t pk[16];
#pragma unroll
      for (int j = 0; j < 16; ++j)
        pk[j] = pack_bf16x2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
      store_box(tmap_out, stg, nbox, pk, t.n * kBN + c * 32, box_row, lane);
    } else if (rv && kF32) {
      uint4* dst = reinterpret_cast<uint4*>(p.out_f32 + ooff + c * 32);
#pragma unroll
      for (int k = 0; k < 8; ++k) dst[k] = make_uint4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
    } else if (rv) {
      uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        uint4 o;
        o.x = pack_bf16x2(__uint_as_float(v[8 * k + 0]), __uint_as_float(v[8 * k + 1]));
        o.y = pack_bf16x2(__uint_as_float(v[8 * k + 2]), __uint_as_float(v[8 * k + 3]));
        o.z = pack_bf16x2(__uint_as_float(v[8 * k + 4]), __uint_as_float(v[8 * k + 5]));
        o.w = pack_bf16x2(__uint_as_float(v[8 * k + 6]), __uint_as_float(v[8 * k + 7]));
        dst[k] = o;
      }
    }
  };
  const int nch = cols / 32;                      // even: n_out is a multiple of 64
  uint32_t ra[32], rb[32];
  if (t.kblocks == 0) {                           // no tokens: the accumulator was never written
#pragma unroll
    for (int j = 0; j < 32; ++j) ra[j] = 0u;
    for (int c = 0; c < nch; ++c) process(c, ra);
    return;
  }
  // chunk c + 1's TMEM load is in flight while chunk c is stored
  tmem_ld32_issue(taddr, ra);
#pragma unroll 1
  for (int c = 0; c < nch; c += 2) {
    tmem_ld_wait(ra);
    tmem_ld32_issue(taddr + static_cast<uint32_t>((c + 1) * 32), rb);
    process(c, ra);
    tmem_ld_wait(rb);
    if (c + 2 < nch) tmem_ld32_issue(taddr + static_cast<uint32_t>((c + 2) * 32), ra);
    process(c + 1, rb);
  }
}

__device__ __forceinline__ float bf16_at(const uint4& u, int j) {
  const uint32_t w = j < 2 ? u.x : (j < 4 ? u.y : (j < 6 ? u.z : u.w));
  return (j & 1) ? bf16_hi(w) : bf16_lo(w);
}

// dH tile: rows are slots of expert e; acc = dY . W2_e (dY already scaled
// by the gate).  dA = acc where H > 0; dgp[slot, n] = sum_cols acc * H for
// kept slots.  Rows past the capacity belong to the next expert and are not
// touched; rows in [kept, C) have dY = 0, so dA = 0 there.
__device__ __forceinline__ void epi_dh(const BwdParams& p, const CUtensorMap* tmap_out,
                                       const BTile& t, uint32_t taddr, int q, int lane,
                                       uint32_t stg, int& nbox) {
  const int64_t r_in = static_cast<int64_t>(t.m) * kBM + q * 32 + lane;
  // dA of a warp whose 32 rows all lie inside the expert's capacity goes out
  // as TMA box stores; otherwise row by row (rows past C are not written)
  const int64_t rbase = static_cast<int64_t>(t.m) * kBM + q * 32;
  const bool bulk = rbase + 32 <= p.C;
  const int box_row = static_cast<int>(static_cast<int64_t>(t.e) * p.C + rbase);
  const int64_t cnt = p.counts[t.e];
  const int64_t ne = cnt < p.C ? cnt : p.C;
  const bool in_cap = r_in < p.C;
  const bool kept = r_in < ne;
  const int64_t s = static_cast<int64_t>(t.e) * p.C + r_in;
  const int cols = p.n_out - t.n * kBN < kBN ? p.n_out - t.n * kBN : kBN;
  const int64_t off = s * p.n_out + t.n * kBN;
  float dot = 0.f;
  // chunk c + 1's TMEM load and H loads are in flight while chunk c is
  // processed (nch is even: n_out is a multiple of 64)
  const int nch = cols / 32;
  auto load_h = [&](int c, uint4* hv) {
    if (in_cap) {
#pragma unroll
      for (int k = 0; k < 4; ++k) hv[k] = ld_u4(p.h + off + c * 32 + 8 * k);
    }
  };
  auto process = [&](int c, const uint32_t* v, const uint4* hv) {
    if (bulk) {
      uint32_t pk[16];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
          const float d0 = __uint_as_float(v[8 * k + j]), d1 = __uint_as_float(v[8 * k + j + 1]);
          const float h0 = bf16_at(hv[k], j), h1 = bf16_at(hv[k], j + 1);
          if (kept) dot = fmaf(d1, h1, fmaf(d0, h0, dot));
          pk[4 * k + j / 2] = pack_bf16x2(h0 > 0.f ? d0 : 0.f, h1 > 0.f ? d1 : 0.f);
        }
      }
      store_box(tmap_out, stg, nbox, pk, t.n * kBN + c * 32, box_row, lane);
    } else if (in_cap) {
      uint4* dst = reinterpret_cast<uint4*>(p.out + off + c * 32);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float a[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float d = __uint_as_float(v[8 * k + j]);
          const float h = bf16_at(hv[k], j);
          a[j] = h > 0.f ? d : 0.f;
          if (kept) dot = fmaf(d, h, dot);
        }
        uint4 o;
        o.x = pack_bf16x2(a[0], a[1]);
        o.y = pack_bf16x2(a[2], a[3]);
        o.z = pack_bf16x2(a[4], a[5]);
        o.w = pack_bf16x2(a[6], a[7]);
        dst[k] = o;
      }
    }
  };
  uint32_t ra[32], rb[32];
  uint4 ha[4], hb[4];
  tmem_ld32_issue(taddr, ra);
  load_h(0, ha);
#pragma unroll 1
  for (int c = 0; c < nch; c += 2) {
    tmem_ld_wait(ra);
    tmem_ld32_issue(taddr + static_cast<uint32_t>((c + 1) * 32), rb);
    load_h(c + 1, hb);
    process(c, ra, ha);
    tmem_ld_wait(rb);
    if (c + 2 < nch) {
      tmem_ld32_issue(taddr + static_cast<uint32_t>((c + 2) * 32), ra);
      load_h(c + 2, ha);
    }
    process(c + 1, rb, hb);
  }
  if (kept) p.dgp[s * p.ntiles_n + t.n] = dot;
}

// dX tile: rows are slots; kept slots write their token's input gradient
// dx[t] = (residual ? dout[t] : 0) + acc, rounded once (acc holds dA W1_e
// and the router term dh W_r).
__device__ __forceinline__ void epi_dx(const BwdParams& p, const BTile& t, uint32_t taddr, int q,
                                       int lane) {
  const int64_t r_in = static_cast<int64_t>(t.m) * kBM + q * 32 + lane;
  const int64_t cnt = p.counts[t.e];
  const int64_t ne = cnt < p.C ? cnt : p.C;
  const bool kept = r_in < ne;
  const int64_t tok = kept ? p.slot_token[static_cast<int64_t>(t.e) * p.C + r_in] : 0;
  const int cols = p.n_out - t.n * kBN < kBN ? p.n_out - t.n * kBN : kBN;
  const int64_t off = tok * p.n_out + t.n * kBN;
  for (int c = 0; c < cols / 32; ++c) {
    uint32_t v[32];
    tmem_ld32_issue(taddr + static_cast<uint32_t>(c * 32), v);
    tmem_ld_wait(v);
    if (kept) {
      uint4* dst = reinterpret_cast<uint4*>(p.dx + off + c * 32);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int64_t o8 = off + c * 32 + 8 * k;
        float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (p.residual) {
          const uint4 g = ld_u4(p.dout + o8);
#pragma unroll
          for (int j = 0; j < 8; ++j) a[j] += bf16_at(g, j);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) a[j] += __uint_as_float(v[8 * k + j]);
        uint4 o;
        o.x = pack_bf16x2(a[0], a[1]);
        o.y = pack_bf16x2(a[2], a[3]);
        o.z = pack_bf16x2(a[4], a[5]);
        o.w = pack_bf16x2(a[6], a[7]);
        dst[k] = o;
      }
    }
  }
}

// dX tile for top-2: kept slot rows store their fp32 accumulator (dA W1_e
// plus the router term where the slot carries it) at the slot; the token's
// sum over its slots and the residual are added by a later kernel.
__device__ __forceinline__ void epi_dx_slot(const BwdParams& p, const BTile& t, uint32_t taddr,
                                            int q, int lane) {
  const int64_t r_in = static_cast<int64_t>(t.m) * kBM + q * 32 + lane;
  const int64_t cnt = p.counts[t.e];
  const int64_t ne = cnt < p.C ? cnt : p.C;
  const bool kept = r_in < ne;
  const int cols = p.n_out - t.n * kBN < kBN ? p.n_out - t.n * kBN : kBN;
  const int64_t off = (static_cast<int64_t>(t.e) * p.C + r_in) * p.n_out + t.n * kBN;
  for (int c = 0; c < cols / 32; ++c) {
    uint32_t v[32];
    tmem_ld32_issue(taddr + static_cast<uint32_t>(c * 32), v);
    tmem_ld_wait(v);
    if (kept) {
      uint4* dst = reinterpret_cast<uint4*>(p.out_f32 + off + c * 32);
#pragma unroll
      for (int k = 0; k < 8; ++k) dst[k] = make_uint4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
    }
  }
}

}  // namespace

template <int kSched, int kEpi>
__global__ void __launch_bounds__(kBwdThreads, 1) bwd_gemm_kernel(
    const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
    const __grid_constant__ CUtensorMap tmap_a2, const __grid_constant__ CUtensorMap tmap_b2,
    BwdParams p) {
  constexpr bool kAMN = kSched != kSchedRows;       // rows: A K-major; else A MN-major
  const int total = kSched == kSchedRows ? p.mtile_start[p.N] * p.ntiles_n
                                         : p.N * p.ntiles_m * p.ntiles_n;
  if (static_cast<int>(blockIdx.x) >= total) return;    // uniform for the block

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* stage_out = smem + kBwdStages * kBwdStageBytes;       // [4 warps][2 boxes x 2 KB]
  uint8_t* tail = stage_out + 4 * 4096;
  uint64_t* full = reinterpret_cast<uint64_t*>(tail);
  uint64_t* empty = full + kBwdStages;
  uint64_t* tfull = empty + kBwdStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int* mts = reinterpret_cast<int*>(tail + 128);                      // [N + 1]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long lim = p.spin;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kBwdStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (kSched == kSchedRows)
    for (int i = threadIdx.x; i <= p.N; i += blockDim.x) mts[i] = p.mtile_start[i];
  if (warp == 1) {
    tmem_alloc(tmem_holder, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmap_a);
      tma_prefetch_desc(&tmap_b);
      const int kmain = p.K / kBK;
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_phase = 0;
      for (int tile = blockIdx.x; tile < total && !*abort_flag; tile += gridDim.x) {
        const BTile t = bwd_tile<kSched>(p, mts, tile);
        bool ok = true;
        for (int kb = 0; kb < t.kblocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, lim)) {
            report_error(p.err, SWITCH_ERR_TIMEOUT, kWhereGemmProducer, tile);
            *abort_flag = 1;
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * kBwdStageBytes;
          uint8_t* sb = sa + kABytes;
          mbar_arrive_expect_tx(&full[stage], kBwdStageBytes);
          const int slot0 = static_cast<int>(static_cast<int64_t>(t.e) * p.C + t.m * kBM);
          if (kSched == kSchedRows && kb < kmain) {
            // A: 128 slot rows x 64 K, K-major; B: MN-major boxes of the
            // expert's weight rows kb*64.. (64 K rows x 64 output columns)
            tma_load_2d(sa, &tmap_a, &full[stage], kb * kBK, slot0);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              tma_load_2d(sb + j * kBox, &tmap_b, &full[stage], t.n * kBN + 64 * j,
                          t.e * p.b_rows + kb * kBK);
          } else if (kSched == kSchedRows) {
            // extra terms (hi.hi, lo.hi, hi.lo) from [2][rows][K] planes
            const int x = kb - kmain;
            const int term = x / p.kx_blocks;
            const int kk = x - term * p.kx_blocks;
            tma_load_3d(sa, &tmap_a2, &full[stage], kk * kBK, slot0, term == 1 ? 1 : 0);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              tma_load_3d(sb + j * kBox, &tmap_b2, &full[stage], t.n * kBN + 64 * j, kk * kBK,
                          term == 2 ? 1 : 0);
          } else if (kSched == kSchedSplit) {
            // A: MN-major boxes of plane `term`, rows chunk*len + kb*64..;
            // B: MN-major boxes of the same rows
            const int term = t.e / p.nsplit;
            const int row = static_cast<int>(static_cast<int64_t>(t.e % p.nsplit) * p.split_len) +
                            kb * kBK;
#pragma unroll
            for (int j = 0; j < 2; ++j)
              tma_load_3d(sa + j * kBox, &tmap_a, &full[stage], t.m * kBM + 64 * j, row, term);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              tma_load_2d(sb + j * kBox, &tmap_b, &full[stage], t.n * kBN + 64 * j, row);
          } else {
            // both operands MN-major from [N][C][inner] maps: K = slots
#pragma unroll
            for (int j = 0; j < 2; ++j)
              tma_load_3d(sa + j * kBox, &tmap_a, &full[stage], t.m * kBM + 64 * j, kb * kBK,
                          t.e);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              tma_load_3d(sb + j * kBox, &tmap_b, &full[stage], t.n * kBN + 64 * j, kb * kBK,
                          t.e);
          }
          issued_mask |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == kBwdStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
      }
      // Never leave with copies in flight into this CTA's shared memory.
      for (int s = 0; s < kBwdStages; ++s)
        if (((issued_mask >> s) & 1u) &&
            !mbar_wait(&full[s], (issued_phase >> s) & 1u, kDefaultSpinCycles))
          report_error(p.err, SWITCH_ERR_TIMEOUT, kWhereDrain, s);
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32_major(kBM, kBN, kAMN, true);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool any = false;
      for (int tile = blockIdx.x; tile < total && !*abort_flag; tile += gridDim.x) {
        const BTile t = bwd_tile<kSched>(p, mts, tile);
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, lim)) {
          report_error(p.err, SWITCH_ERR_TIMEOUT, kWhereGemmMma, tile);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kBN);
        bool ok = true;
        for (int kb = 0; kb < t.kblocks; ++kb) {
          if (!mbar_wait(&full[stage], phase, lim)) {
            report_error(p.err, SWITCH_ERR_TIMEOUT, kWhereGemmMma, tile);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * kBwdStageBytes);
          const uint32_t sb = sa + kABytes;
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            const uint64_t ad = kAMN ? sw128_mnmajor_desc(sa + k * 2048, kBox)
                                     : sw128_kmajor_desc(sa + k * 32);
            umma_bf16(d_tmem, ad, sw128_mnmajor_desc(sb + k * 2048, kBox), idesc,
                      (kb | k) != 0 ? 1u : 0u);
          }
          any = true;
          umma_commit(&empty[stage]);
          if (++stage == kBwdStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);      // also for an empty K loop (the epilogue writes zeros)
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (any && *abort_flag) {
        umma_commit(drain);
        if (!mbar_wait(drain, 0, kDefaultSpinCycles))
          report_error(p.err, SWITCH_ERR_TIMEOUT, kWhereDrain, -1);
      }
    }
  } else {
    // ----------------------------------------------------- epilogue warps
    const int q = warp & 3;            // TMEM lanes 32q..32q+31 (warp rank in its warpgroup)
    const uint32_t stg = smem_u32(stage_out + q * 4096);
    int nbox = 0;                      // running count: the two boxes alternate
    int acc = 0;
    uint32_t acc_phase = 0;
    if (lane == 0 && (kEpi == kEpiDH || kEpi == kEpiStore)) tma_prefetch_desc(&tmap_a2);
    prefetch_epilogue_rows<kEpi>(p, bwd_tile<kSched>(p, mts, blockIdx.x), q, lane);
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      const bool ok = __all_sync(0xffffffffu, mbar_wait_sleepy(&tfull[acc], acc_phase, lim));
      if (!ok) {
        if (lane == 0) {
          report_error(p.err, SWITCH_ERR_TIMEOUT, kWhereGemmEpilogue, tile);
          *abort_flag = 1;
        }
        break;
      }
      tc_fence_after();
      const BTile t = bwd_tile<kSched>(p, mts, tile);
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc * kBN);
      // dH and bf16 stores: tmap_a2 is the output's box-store map
      if (kEpi == kEpiStore) epi_store<false>(p, &tmap_a2, t, taddr, q, lane, stg, nbox);
      else if (kEpi == kEpiStoreF32) epi_store<true>(p, &tmap_a2, t, taddr, q, lane, stg, nbox);
      else if (kEpi == kEpiDH) epi_dh(p, &tmap_a2, t, taddr, q, lane, stg, nbox);
      else if (kEpi == kEpiDXSlot) epi_dx_slot(p, t, taddr, q, lane);
      else epi_dx(p, t, taddr, q, lane);
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      if (tile + static_cast<int>(gridDim.x) < total)
        prefetch_epilogue_rows<kEpi>(p, bwd_tile<kSched>(p, mts, tile + gridDim.x), q, lane);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    if (lane == 0) bulk_wait_all();    // boxes stored from shared memory are written
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

// ------------------------------------------------- weight gradients, CTA pairs
//
// dW_e = A_e^T B_e with both operands MN-major, as the weight schedule above,
// on 256 x 256 pair tiles: CTA r of the pair loads output rows
// m*256 + 128 r .. + 127 of A and output columns n*256 + 128 r .. + 127 of B
// (two 64 x 64 boxes each, 32 KB per K step, completing on the leader's
// barrier; no copy is multicast); the leader issues
// tcgen05.mma.cta_group::2 (M = 256, N = 256) and each CTA's TMEM holds its
// 128 rows.  Per SM that is 32 KB of operands per K step instead of 48 KB
// for the same tensor work.
constexpr int kPairBwdStages = 6;
constexpr uint32_t kPairBwdStageBytes = 4 * kBox;       // 2 A boxes + 2 B boxes

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kBwdThreads, 1)
    bwd_wgrad_pair_kernel(const __grid_constant__ CUtensorMap tmap_a,
                          const __grid_constant__ CUtensorMap tmap_b,
                          const __grid_constant__ CUtensorMap tmap_out, BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* stage_out = smem + kPairBwdStages * kPairBwdStageBytes;   // [4 warps][2 x 2 KB]
  uint8_t* tail = stage_out + 4 * 4096;
  uint64_t* full = reinterpret_cast<uint64_t*>(tail);    // leader: both CTAs' TMA bytes
  uint64_t* empty = full + kPairBwdStages;               // local: stage free (MMA done)
  uint64_t* tfull = empty + kPairBwdStages;              // local: accumulator ready
  uint64_t* tempty = tfull + 2;                          // leader: accumulator drained
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cid = static_cast<int>(cluster_id_x());
  const int ncl = static_cast<int>(cluster_count_x());
  const long long lim = p.spin;
  const int tm2 = (p.M_out + 2 * kBM - 1) / (2 * kBM);   // 256-row tiles per expert
  const int total = p.N * tm2 * p.ntiles_n;
  if (cid >= total) return;                 // same decision in both CTAs of the pair

  // pair tile -> (expert, 256-row tile, 256-column tile, K blocks)
  auto tile_of = [&](int t) {
    BTile r;
    const int per = tm2 * p.ntiles_n;
    r.e = t / per;
    const int local = t - r.e * per;
    r.n = local / tm2;
    r.m = local - r.n * tm2;
    const int64_t cnt = p.counts[r.e];
    const int64_t ne = cnt < p.C ? cnt : p.C;
    r.kblocks = static_cast<int>((ne + kBK - 1) / kBK);
    return r;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairBwdStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 8);             // 4 epilogue warps x 2 CTAs
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();                           // the peer's barriers exist before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const uint32_t full_lead = map_to_rank(smem_u32(full), 0);
  const uint32_t tempty_lead = map_to_rank(smem_u32(tempty), 0);

  if (warp == 0) {
    // ------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmap_a);
      tma_prefetch_desc(&tmap_b);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_phase = 0;
      for (int tile = cid; tile < total && !*abort_flag; tile += ncl) {
        const BTile t = tile_of(tile);
        const int a0 = t.m * 2 * kBM + static_cast<int>(rank) * kBM;
        const int b0 = t.n * kBN + static_cast<int>(rank) * kBM;
        bool ok = true;
        for (int kb = 0; kb < t.kblocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, lim)) {
            report_error(p.err, SWITCH_ERR_TIMEOUT, kWhereGemmProducer, tile);
            *abort_flag = 1;
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * kPairBwdStageBytes;
          uint8_t* sb = sa + 2 * kBox;
          const uint32_t bar = full_lead + 8u * stage;
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * kPairBwdStageBytes);
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            tma_load_3d_pair(sa + j * kBox, &tmap_a, bar, a0 + 64 * j, kb * kBK, t.e);
            tma_load_3d_pair(sb + j * kBox, &tmap_b, bar, b0 + 64 * j, kb * kBK, t.e);
          }
          issued_mask |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == kPairBwdStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
      }
      // both CTAs' TMA bytes complete on the leader's barriers, which the
      // leader drains before the final cluster barrier
      if (leader) {
        for (int s = 0; s < kPairBwdStages; ++s)
          if (((issued_mask >> s) & 1u) &&
              !mbar_wait_cluster(&full[s], (issued_phase >> s) & 1u, kDefaultSpinCycles))
            report_error(p.err, SWITCH_ERR_TIMEOUT, kWhereDrain, s);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------- MMA issuer (leader)
    if (leader && lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32_major(2 * kBM, kBN, true, true);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool any = false;
      for (int tile = cid; tile < total && !*abort_flag; tile += ncl) {
        const BTile t = tile_of(tile);
        if (!mbar_wait_cluster(&tempty[acc], acc_phase ^ 1u, lim)) {
          report_error(p.err, SWITCH_ERR_TIMEOUT, kWhereGemmMma, tile);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kBN);
        bool ok = true;
        for (int kb = 0; kb < t.kblocks; ++kb) {
          if (!mbar_wait_cluster(&full[stage], phase, lim)) {
            report_error(p.err, SWITCH_ERR_TIMEOUT, kWhereGemmMma, tile);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * kPairBwdStageBytes);
          const uint32_t sb = sa + 2 * kBox;
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)
            umma_bf16_pair(d_tmem, sw128_mnmajor_desc(sa + k * 2048, kBox),
                           sw128_mnmajor_desc(sb + k * 2048, kBox), idesc,
                           (kb | k) != 0 ? 1u : 0u);
          any = true;
          umma_commit_pair(&empty[stage], 0x3);
          if (++stage == kPairBwdStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit_pair(&tfull[acc], 0x3);   // also for an empty K loop (zeros written)
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (any && *abort_flag) {
        umma_commit_pair(drain, 0x1);
        if (!mbar_wait(drain, 0, kDefaultSpinCycles))
          report_error(p.err, SWITCH_ERR_TIMEOUT, kWhereDrain, -1);
      }
    }
  } else {
    // ----------------------------------------------------- epilogue warps
    const int q = warp & 3;
    const uint32_t stg = smem_u32(stage_out + q * 4096);
    int nbox = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    if (lane == 0) tma_prefetch_desc(&tmap_out);
    for (int tile = cid; tile < total; tile += ncl) {
      const bool ok = __all_sync(0xffffffffu, mbar_wait_sleepy(&tfull[acc], acc_phase, lim));
      if (!ok) {
        if (lane == 0) {
          report_error(p.err, SWITCH_ERR_TIMEOUT, kWhereGemmEpilogue, tile);
          *abort_flag = 1;
        }
        break;
      }
      tc_fence_after();
      BTile t = tile_of(tile);
      t.m = 2 * t.m + static_cast<int>(rank);     // this CTA's 128-row half
      epi_store<false>(p, &tmap_out, t,
                       tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                           static_cast<uint32_t>(acc * kBN),
                       q, lane, stg, nbox);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader) mbar_arrive(&tempty[acc]);
        else mbar_arrive_remote(tempty_lead + 8u * acc);
      }
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    if (lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();                           // no CTA leaves while its peer may still signal it
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, kTmemCols);
}

// ------------------------------------------------------------------- host

// 3-D bf16 tensor [outer][mid][inner] (inner contiguous), 128-byte swizzle,
// box box_inner x box_mid x 1; out-of-range elements read as zero.
bool make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t mid,
                       uint64_t outer, uint32_t box_inner, uint32_t box_mid) {
  PFN_encodeTiled enc = get_encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[3] = {inner, mid, outer};
  const cuuint64_t strides[2] = {inner * 2, inner * mid * 2};
  const cuuint32_t box[3] = {box_inner, box_mid, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

template <int kSched, int kEpi>
static cudaError_t run_bwd(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& ta2,
                           const CUtensorMap& tb2, const BwdParams& p, int num_sms,
                           cudaStream_t st) {
  const size_t smem =
      1024 + kBwdStages * kBwdStageBytes + 4 * 4096 + 128 + sizeof(int) * (p.N + 1);
  static size_t smem_set[64] = {};
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(&bwd_gemm_kernel<kSched, kEpi>),
                                    smem, smem_set);
  if (e != cudaSuccess) return e;
  bwd_gemm_kernel<kSched, kEpi><<<num_sms, kBwdThreads, smem, st>>>(ta, tb, ta2, tb2, p);
  return cudaGetLastError();
}

static cudaError_t run_wgrad_pair(const CUtensorMap& ta, const CUtensorMap& tb,
                                  const CUtensorMap& to, const BwdParams& p, int num_sms,
                                  cudaStream_t st) {
  const size_t smem = 1024 + kPairBwdStages * kPairBwdStageBytes + 4 * 4096 + 256;
  static size_t smem_set[64] = {};
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(&bwd_wgrad_pair_kernel), smem,
                                    smem_set);
  if (e != cudaSuccess) return e;
  bwd_wgrad_pair_kernel<<<(num_sms / 2) * 2, kBwdThreads, smem, st>>>(ta, tb, to, p);
  return cudaGetLastError();
}

static BwdParams base_params(const BwdFfnArgs& a) {
  BwdParams p{};
  p.N = a.N;
  p.C = a.C;
  p.counts = a.counts;
  p.mtile_start = a.mtile_start;
  p.slot_token = a.slot_token;
  p.err = a.err;
  p.spin = a.spin;
  return p;
}

cudaError_t launch_bwd_dh(const BwdFfnArgs& a, cudaStream_t st) {
  const uint64_t slots = static_cast<uint64_t>(a.N) * static_cast<uint64_t>(a.C);
  CUtensorMap ta, tb, to;
  bool ok = make_tmap_bf16_2d(&ta, a.dys, a.d, slots, kBK, kBM);
  ok = ok && make_tmap_bf16_2d(&tb, a.w2, a.F, static_cast<uint64_t>(a.N) * a.d, 64, 64);
  ok = ok && make_tmap_bf16_2d(&to, a.da, a.F, slots, 32, 32, true);    // dA box stores
  if (!ok) return cudaErrorInvalidValue;
  BwdParams p = base_params(a);
  p.K = a.d;
  p.n_out = a.F;
  p.ntiles_n = (a.F + kBN - 1) / kBN;
  p.b_rows = a.d;
  p.h = static_cast<const __nv_bfloat16*>(a.hbuf);
  p.out = static_cast<__nv_bfloat16*>(a.da);
  p.dgp = a.dgp;
  return run_bwd<kSchedRows, kEpiDH>(ta, tb, to, tb, p, a.num_sms, st);
}

cudaError_t launch_bwd_dw(const BwdFfnArgs& a, cudaStream_t st) {
  CUtensorMap ta2, tb2, ta1, tb1, to2, to1;
  const uint64_t C = static_cast<uint64_t>(a.C), N = static_cast<uint64_t>(a.N);
  // weight-gradient box stores: dW2 [N*d, F], dW1 [N*F, d]
  bool okb = make_tmap_bf16_2d(&to2, a.dw2, a.F, N * a.d, 32, 32, true);
  okb = okb && make_tmap_bf16_2d(&to1, a.dw1, a.d, N * a.F, 32, 32, true);
  if (!okb) return cudaErrorInvalidValue;
  bool ok = make_tmap_bf16_3d(&ta2, a.dys, a.d, C, N, 64, kBK);
  ok = ok && make_tmap_bf16_3d(&tb2, a.hbuf, a.F, C, N, 64, kBK);
  ok = ok && make_tmap_bf16_3d(&ta1, a.da, a.F, C, N, 64, kBK);
  ok = ok && make_tmap_bf16_3d(&tb1, a.x_disp, a.d, C, N, 64, kBK);
  if (!ok) return cudaErrorInvalidValue;
  if (a.pair_dw) {
    // the A maps' boxes are 64 rows of the 128-row half each CTA loads
    BwdParams q2 = base_params(a);
    q2.M_out = a.d;
    q2.n_out = a.F;
    q2.ntiles_n = (a.F + kBN - 1) / kBN;
    q2.out = static_cast<__nv_bfloat16*>(a.dw2);
    cudaError_t e = run_wgrad_pair(ta2, tb2, to2, q2, a.num_sms, st);
    if (e != cudaSuccess) return e;
    BwdParams q1 = base_params(a);
    q1.M_out = a.F;
    q1.n_out = a.d;
    q1.ntiles_n = (a.d + kBN - 1) / kBN;
    q1.out = static_cast<__nv_bfloat16*>(a.dw1);
    return run_wgrad_pair(ta1, tb1, to1, q1, a.num_sms, st);
  }
  // dW2_e [d, F] = dY_e^T H_e
  BwdParams p2 = base_params(a);
  p2.M_out = a.d;
  p2.n_out = a.F;
  p2.ntiles_m = (a.d + kBM - 1) / kBM;
  p2.ntiles_n = (a.F + kBN - 1) / kBN;
  p2.out = static_cast<__nv_bfloat16*>(a.dw2);
  cudaError_t e = run_bwd<kSchedWeight, kEpiStore>(ta2, tb2, to2, tb2, p2, a.num_sms, st);
  if (e != cudaSuccess) return e;
  // dW1_e [F, d] = dA_e^T X_e
  BwdParams p1 = base_params(a);
  p1.M_out = a.F;
  p1.n_out = a.d;
  p1.ntiles_m = (a.F + kBM - 1) / kBM;
  p1.ntiles_n = (a.d + kBN - 1) / kBN;
  p1.out = static_cast<__nv_bfloat16*>(a.dw1);
  return run_bwd<kSchedWeight, kEpiStore>(ta1, tb1, to1, tb1, p1, a.num_sms, st);
}

cudaError_t launch_bwd_dx(const BwdFfnArgs& a, cudaStream_t st) {
  const uint64_t slots = static_cast<uint64_t>(a.N) * static_cast<uint64_t>(a.C);
  CUtensorMap ta, tb, ta2, tb2;
  bool ok = make_tmap_bf16_2d(&ta, a.da, a.F, slots, kBK, kBM);
  ok = ok && make_tmap_bf16_2d(&tb, a.w1, a.d, static_cast<uint64_t>(a.N) * a.F, 64, 64);
  // router term: dh planes per slot [2][slots][Np] (K-major, 128-row boxes)
  // and W_r planes [2][Np][d] (MN-major 64 x 64 boxes; rows N..Np-1 zero)
  ok = ok && make_tmap_bf16_3d(&ta2, a.dhs, a.n_pad, slots, 2, kBK, kBM);
  ok = ok && make_tmap_bf16_3d(&tb2, a.wrp, a.d, a.n_pad, 2, 64, kBK);
  if (!ok) return cudaErrorInvalidValue;
  BwdParams p = base_params(a);
  p.K = a.F;
  p.n_out = a.d;
  p.ntiles_n = (a.d + kBN - 1) / kBN;
  p.b_rows = a.F;
  p.kx_blocks = a.n_pad / kBK;
  p.kx_terms = 3;
  p.dout = static_cast<const __nv_bfloat16*>(a.dout);
  p.dx = static_cast<__nv_bfloat16*>(a.dx);
  p.residual = a.residual ? 1 : 0;
  if (a.dxs) {
    p.out_f32 = a.dxs;
    return run_bwd<kSchedRows, kEpiDXSlot>(ta, tb, ta2, tb2, p, a.num_sms, st);
  }
  return run_bwd<kSchedRows, kEpiDX>(ta, tb, ta2, tb2, p, a.num_sms, st);
}

// Token chunks per term: about one wave of tiles over a B200's 148 SMs (a
// fixed count, so the scratch size does not depend on the device).
static int split_chunks(int64_t T, int N, int d, int /*num_sms*/) {
  const int tiles = ((N + kBM - 1) / kBM) * ((d + kBN - 1) / kBN);
  int nch = 148 / (2 * tiles);
  if (nch < 1) nch = 1;
  const int64_t max_ch = (T + kBK - 1) / kBK;
  return static_cast<int>(nch < max_ch ? nch : max_ch);
}

size_t router_bwd_tc_part_floats(int64_t T, int N, int d, int num_sms) {
  return static_cast<size_t>(2 * split_chunks(T, N, d, num_sms)) * N * static_cast<size_t>(d);
}

// dw_r[j] = sum over batches b of part[b][j] in order (loads issued eight
// at a time, additions in batch order).
__global__ void split_reduce_kernel(int nb, int64_t nd, const float* __restrict__ part,
                                    float* __restrict__ dw_r) {
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j >= nd) return;
  float s = 0.f;
  int b = 0;
  for (; b + 8 <= nb; b += 8) {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = __ldg(part + (b + u) * nd + j);
#pragma unroll
    for (int u = 0; u < 8; ++u) s += v[u];
  }
  for (; b < nb; ++b) s += part[b * nd + j];
  dw_r[j] = s;
}

// db[i] = sum over the per-tile column sums colsum[p][i], p in order: one
// warp per expert, lanes take parts p = lane + 32 q in turn and the 32 lane
// sums are added in a fixed butterfly.
__global__ void colsum_reduce_kernel(int nparts, int N, const float* __restrict__ colsum,
                                     float* __restrict__ db) {
  const int i = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (i >= N) return;
  float s = 0.f;
  for (int p = lane; p < nparts; p += 32) s += colsum[static_cast<int64_t>(p) * N + i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) db[i] = s;
}

cudaError_t launch_router_bwd_dw_tc(int64_t T, int N, int Np, int d, const void* dhp,
                                    const void* x, float* part, const float* colsum,
                                    float* dw_r, float* db, DevErr* err, long long spin,
                                    int num_sms, cudaStream_t st) {
  const int nch = split_chunks(T, N, d, num_sms);
  int64_t len = (T + nch - 1) / nch;
  len = (len + kBK - 1) / kBK * kBK;
  CUtensorMap ta, tb;
  bool ok = make_tmap_bf16_3d(&ta, dhp, Np, T, 2, 64, kBK);
  ok = ok && make_tmap_bf16_2d(&tb, x, d, T, 64, kBK);
  if (!ok) return cudaErrorInvalidValue;
  BwdParams p{};
  p.N = 2 * nch;                  // batches: term * nch + chunk
  p.M_out = N;
  p.n_out = d;
  p.ntiles_m = (N + kBM - 1) / kBM;
  p.ntiles_n = (d + kBN - 1) / kBN;
  p.nsplit = nch;
  p.split_len = len;
  p.split_rows = T;
  p.out_f32 = part;
  p.err = err;
  p.spin = spin;
  cudaError_t e = run_bwd<kSchedSplit, kEpiStoreF32>(ta, tb, ta, tb, p, num_sms, st);
  if (e != cudaSuccess) return e;
  const int64_t nd = static_cast<int64_t>(N) * d;
  const int nparts = static_cast<int>((T + 127) / 128);
  split_reduce_kernel<<<static_cast<unsigned>((nd + 255) / 256), 256, 0, st>>>(2 * nch, nd, part,
                                                                             dw_r);
  e = cudaGetLastError();
  if (e != cudaSuccess || db == nullptr) return e;
  colsum_reduce_kernel<<<static_cast<unsigned>((N + 7) / 8), 256, 0, st>>>(nparts, N, colsum, db);
  return cudaGetLastError();
}

}  // namespace smoe
