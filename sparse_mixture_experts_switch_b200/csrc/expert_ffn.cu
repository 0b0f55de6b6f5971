// Expert FFNs over the capacity buffers: N independent ReLU FFNs
// ("Switch Transformers: scaling to trillion-parameter models", section
// "The Core Idea"), each applied to the tokens that hold its slots
// (section "Expert Capacity and the Capacity Factor"), and optionally the
// gate-scaled combine with the residual fused into the second GEMM's
// epilogue (section "Switch Routing: From Top-k to k = 1", combine
// equation; one writer per output row since k = 1).
//
// bf16 path: a persistent tcgen05 grouped GEMM.
//   * tile = 128 slots (rows) x 256 output columns, K in blocks of 64;
//   * warp 0 feeds a 4-stage shared-memory ring: weights (B) by TMA with
//     the 128-byte swizzle; in GEMM1 the A rows are gathered straight from x
//     through slot_token by the warp's 32 lanes with 16-byte cp.async into
//     the same swizzled layout (the next tile's token ids are fetched while
//     the current tile streams), so the dispatched tokens are never
//     materialised; GEMM2 reads the hidden rows by TMA;
//   * warp 1 issues tcgen05.mma (M=128, N=256, K=16) into one of two TMEM
//     accumulators (2 x 256 fp32 columns) so the epilogue of one tile
//     overlaps the main loop of the next;
//   * warps 2-5 drain TMEM (one token row per thread) through a per-warp
//     shared buffer that turns row-per-thread values into coalesced stores:
//     ReLU + bf16 for the hidden activation, bf16 for Y, or x + gate * acc
//     for the combine;
//   * the tile list comes from device-side counts (no host sync); experts'
//     empty capacity tiles are never scheduled; consecutive CTAs take the
//     M tiles of the same (expert, N tile) so each weight tile is read from
//     HBM about once and from L2 by the rest.
// fp32 path: CUDA-core FMA tiles (no TF32), same tile list semantics.
#include <cstring>

#include "gemm_common.cuh"

namespace smoe {

// ----------------------------------------------------------- tensor maps

PFN_encodeTiled get_encode_fn() {
  static PFN_encodeTiled fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_encodeTiled>(p);
  }
  return fn;
}

// 2-D bf16 tensor [outer, inner] (inner contiguous), 128-byte swizzle by
// default; out-of-range elements read as zero and are never written.
bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                       uint32_t box_inner, uint32_t box_outer, bool swizzle64) {
  PFN_encodeTiled enc = get_encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner * 2};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             swizzle64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ================================================== tcgen05 grouped GEMM

constexpr int kStages = 4;
constexpr uint32_t kStageBytes = kABytes + kBBytes;     // 48 KB

template <bool kGather>
__global__ void __launch_bounds__(kGemmThreads, 1) expert_gemm_kernel(
    const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
    const __grid_constant__ CUtensorMap tmap_out, GemmParams p) {
  const int total = p.mtile_start[p.N] * p.ntiles_n;
  if (static_cast<int>(blockIdx.x) >= total) return;    // uniform for the block

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* stage_out = smem + kStages * kStageBytes;                 // [4][4 KB], 1024-aligned
  uint8_t* tail = stage_out + 4 * kStageOutBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(tail);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int* tok_s = reinterpret_cast<int*>(tail + 128);                    // [4][32]
  int* mts = reinterpret_cast<int*>(tail + 128 + 4 * 32 * 4);         // [N + 1]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long lim = p.spin;
  const int kblocks = p.K / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      // gather mode: one cp.async arrival per gathering lane + the B copy
      mbar_init(&full[s], kGather ? kGatherLanes + 1 : 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  for (int i = threadIdx.x; i <= p.N; i += blockDim.x) mts[i] = p.mtile_start[i];
  if (warp == 1) {
    tmem_alloc(tmem_holder, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0 || warp >= 6) {
    // --------------------------------------------------- producer warps
    // B (weights) by TMA from warp 0; A by TMA (tiled), or in gather mode by
    // the lanes of warps 0, 6, 7, 8 with 16-byte cp.async, 32 rows per warp;
    // lane = (row lane / 8 within a group of 4 rows, 16-byte chunk lane % 8),
    // so one instruction reads four whole 128-byte row segments, and each
    // chunk lands where the 128-byte swizzle puts it (chunk ^ row % 8).
    const bool lead = warp == 0;
    if (!kGather && !lead) goto producer_done;
    {
      if (lead && lane == 0 && !kGather) tma_prefetch_desc(&tmap_a);
      if (lead && lane == 0) tma_prefetch_desc(&tmap_b);
      const int ch = lane & 7;
      const int gw = lead ? 0 : warp - 5;                      // 0..3
      const int row0 = 32 * gw + (lane >> 3);                  // rows row0 + 4 j, j < 8
      const uint32_t vec_per_row = static_cast<uint32_t>(p.K / 8);   // 16-byte units
      // per-lane shared-memory offsets of the 16 rows (two swizzle phases)
      const uint32_t sw_even = static_cast<uint32_t>((ch ^ (row0 & 7)) << 4);
      const uint32_t sw_odd = static_cast<uint32_t>((ch ^ ((row0 + 4) & 7)) << 4);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_phase = 0;
      // 16-byte-unit offset of each row's token in x (~0u: padding row)
      uint32_t roff[8];
      auto load_rows = [&](int t_tile, uint32_t* dst) {
        int e, m, n;
        decode_tile(t_tile, mts, p.N, p.ntiles_n, e, m, n);
        const int64_t n_e = kept_rows(p, e);
        const int64_t slot0 = static_cast<int64_t>(e) * p.C + static_cast<int64_t>(m) * kBM;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int r = row0 + 4 * j;
          dst[j] = (static_cast<int64_t>(m) * kBM + r < n_e)
                       ? static_cast<uint32_t>(p.slot_token[slot0 + r]) * vec_per_row
                       : ~0u;
        }
      };
      if (kGather) load_rows(blockIdx.x, roff);
      for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
        if (__shfl_sync(0xffffffffu, *abort_flag, 0)) break;   // warp-uniform
        int e, m, n;
        decode_tile(tile, mts, p.N, p.ntiles_n, e, m, n);
        const int64_t slot0 = static_cast<int64_t>(e) * p.C + static_cast<int64_t>(m) * kBM;
        uint32_t roff_next[8];
        const int next = tile + gridDim.x;
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
          uint8_t* sa = smem + stage * kStageBytes;
          uint8_t* sb = sa + kABytes;
          if (kGather) {
            const uint4* src0 = reinterpret_cast<const uint4*>(p.a_rows) + kb * 8 + ch;
            const uint32_t dst0 = smem_u32(sa) + static_cast<uint32_t>(row0 * 128);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              if (roff[j] != ~0u)
                cp_async16_s(dst0 + j * 512 + ((j & 1) ? sw_odd : sw_even), src0 + roff[j]);
            }
            cp_async_mbar_arrive_noinc(&full[stage]);
            if (lead && lane == 0) {
              mbar_arrive_expect_tx(&full[stage], kBBytes);
              tma_load_2d(sb, &tmap_b, &full[stage], kb * kBK, e * p.n_out + n * kBN);
            }
          } else if (lane == 0) {
            mbar_arrive_expect_tx(&full[stage], kStageBytes);
            tma_load_2d(sa, &tmap_a, &full[stage], kb * kBK, static_cast<int>(slot0));
            tma_load_2d(sb, &tmap_b, &full[stage], kb * kBK, e * p.n_out + n * kBN);
          }
          issued_mask |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if (kGather) {
#pragma unroll
          for (int j = 0; j < 8; ++j) roff[j] = roff_next[j];
        }
      }
      // Never leave with copies in flight into this CTA's shared memory.
      if (kGather) cp_async_wait_all();
      if (lead && lane == 0) {
        for (int s = 0; s < kStages; ++s)
          if (((issued_mask >> s) & 1u) &&
              !mbar_wait(&full[s], (issued_phase >> s) & 1u, kDefaultSpinCycles))
            report_error(p.err, SWITCH_ERR_TIMEOUT, kWhereDrain, s);
      }
    }
  producer_done:;
  } else if (warp == 1) {
    // --------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool any = false;
      for (int tile = blockIdx.x; tile < total && !*abort_flag; tile += gridDim.x) {
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, lim)) {
          report_error(p.err, SWITCH_ERR_TIMEOUT, kWhereGemmMma, tile);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kBN);
        bool ok = true;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&full[stage], phase, lim)) {
            report_error(p.err, SWITCH_ERR_TIMEOUT, kWhereGemmMma, tile);
            *abort_flag = 1;
            ok = false;
            break;
          }
          if (kGather) fence_proxy_async_smem();   // cp.async data -> tensor-core reads
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * kStageBytes);
          const uint32_t sb = sa + kABytes;
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)
            umma_bf16(d_tmem, sw128_kmajor_desc(sa + k * 32), sw128_kmajor_desc(sb + k * 32),
                      idesc, (kb | k) != 0 ? 1u : 0u);
          any = true;
          umma_commit(&empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
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
    // --------------------------------------------------- epilogue warps
    // Each thread owns one accumulator row (TMEM lane).  Per 32-column chunk
    // the row's values (ReLU'd, or scaled by its gate) go through a per-warp
    // shared buffer so that global stores are written 8 rows x 64 bytes per
    // instruction instead of 32 scattered 16-byte pieces.
    const int q = warp & 3;
    const uint32_t stg = smem_u32(stage_out + q * kStageOutBytes);
    int* tokw = tok_s + q * 32;
    int acc = 0;
    uint32_t acc_phase = 0;
    if (lane == 0 && p.mode != kModeCombine) tma_prefetch_desc(&tmap_out);
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
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
      int e, m, n;
      decode_tile(tile, mts, p.N, p.ntiles_n, e, m, n);
      // combine: fetch the next tile's token now, prefetch its residual row
      // after this tile (the next tile's main loop then hides the latency)
      int ntok = -1, nn = 0;
      if (p.mode == kModeCombine) {
        if (tile == static_cast<int>(blockIdx.x)) prefetch_residual(p, combine_row_token(p, e, m, q, lane), n);
        const int nt = tile + gridDim.x;
        if (nt < total) {
          int e2, m2;
          decode_tile(nt, mts, p.N, p.ntiles_n, e2, m2, nn);
          ntok = combine_row_token(p, e2, m2, q, lane);
        }
      }
      epilogue_tile(p, &tmap_out, e, m, n,
                    tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                        static_cast<uint32_t>(acc * kBN),
                    stg, tokw, q, lane);
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      prefetch_residual(p, ntok, nn);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    if (lane == 0) bulk_wait_all();        // boxes stored from shared memory are written
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

static size_t gemm_smem_bytes(int N) {
  return 1024 + kStages * kStageBytes + kTailBytes + sizeof(int) * (N + 1);
}

template <bool kGather>
static cudaError_t run_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& to,
                            const GemmParams& gp, int num_sms, cudaStream_t st) {
  const size_t smem = gemm_smem_bytes(gp.N);
  static size_t smem_set[64] = {};
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(&expert_gemm_kernel<kGather>), smem, smem_set);
  if (e != cudaSuccess) return e;
  expert_gemm_kernel<kGather><<<num_sms, kGemmThreads, smem, st>>>(ta, tb, to, gp);
  return cudaGetLastError();
}

cudaError_t launch_expert_ffn_bf16(const FfnArgs& a, cudaStream_t st) {
  const uint64_t slots = static_cast<uint64_t>(a.N) * static_cast<uint64_t>(a.C);
  CUtensorMap ta1, tb1, ta2, tb2, to1, to2;
  // 64- and 32-row boxes of the token rows (half tiles; ragged pair tiles)
  CUtensorMap ta1h, ta1q, ta2h, ta2q;
  const bool gather = a.x_disp == nullptr;
  const bool rows1 = a.pair1_rows && !gather;   // row-major pairs read rows by TMA only
  // CTA pairs load half a weight tile each (128 rows); single CTAs all 256.
  const uint32_t b_rows1 = (a.pair1 || rows1) ? 128u : static_cast<uint32_t>(kBN);
  const uint32_t b_rows2 = a.pair2 ? 128u : static_cast<uint32_t>(kBN);
  bool ok = true;
  if (gather) {
    memset(&ta1, 0, sizeof(ta1));          // unused: rows are gathered with cp.async
    memset(&ta1h, 0, sizeof(ta1h));
    memset(&ta1q, 0, sizeof(ta1q));
  } else {
    ok = make_tmap_bf16_2d(&ta1, a.x_disp, a.d, slots, kBK, kBM);
    ok = ok && make_tmap_bf16_2d(&ta1h, a.x_disp, a.d, slots, kBK, kBM / 2);
    ok = ok && make_tmap_bf16_2d(&ta1q, a.x_disp, a.d, slots, kBK, kBM / 4);
  }
  ok = ok && make_tmap_bf16_2d(&tb1, a.w1, a.d, static_cast<uint64_t>(a.N) * a.F, kBK, b_rows1);
  ok = ok && make_tmap_bf16_2d(&ta2, a.hbuf, a.F, slots, kBK, kBM);
  ok = ok && make_tmap_bf16_2d(&ta2h, a.hbuf, a.F, slots, kBK, kBM / 2);
  ok = ok && make_tmap_bf16_2d(&ta2q, a.hbuf, a.F, slots, kBK, kBM / 4);
  ok = ok && make_tmap_bf16_2d(&tb2, a.w2, a.F, static_cast<uint64_t>(a.N) * a.d, kBK, b_rows2);
  // epilogue boxes: 32 rows x 32 columns of H (GEMM1) or Y (GEMM2, unfused)
  ok = ok && make_tmap_bf16_2d(&to1, a.hbuf, a.F, slots, 32, 32, true);
  if (a.mode2 == kModeY)
    ok = ok && make_tmap_bf16_2d(&to2, a.y, a.d, slots, 32, 32, true);
  else
    memset(&to2, 0, sizeof(to2));          // unused: the combine scatters rows by token
  if (!ok) return cudaErrorInvalidValue;

  GemmParams g1{};
  g1.N = a.N;
  g1.n_out = a.F;
  g1.K = a.d;
  g1.ntiles_n = (a.F + kBN - 1) / kBN;
  g1.C = a.C;
  g1.counts = a.counts;
  g1.mtile_start = a.mtile_start;
  g1.slot_token = a.slot_token;
  g1.a_rows = static_cast<const __nv_bfloat16*>(a.x);
  g1.mode = kModeHidden;
  g1.out = static_cast<__nv_bfloat16*>(a.hbuf);
  g1.ldo = a.F;
  g1.err = a.err;
  g1.spin = a.spin;
  cudaError_t e;
  if (rows1)
    e = run_gemm_pair_rows(ta1, ta1h, tb1, to1, g1, a.num_sms, st);
  else if (a.pair1)
    e = gather ? run_gemm_pair<true>(ta1, ta1, ta1, tb1, to1, g1, a.num_sms, st)
               : run_gemm_pair<false>(ta1, ta1h, ta1q, tb1, to1, g1, a.num_sms, st);
  else
    e = gather ? run_gemm<true>(ta1, tb1, to1, g1, a.num_sms, st)
               : run_gemm<false>(ta1, tb1, to1, g1, a.num_sms, st);
  if (e != cudaSuccess || a.gemm1_only) return e;

  GemmParams g2 = g1;
  g2.n_out = a.d;
  g2.K = a.F;
  g2.ntiles_n = (a.d + kBN - 1) / kBN;
  g2.a_rows = nullptr;
  g2.mode = a.mode2;
  g2.out = static_cast<__nv_bfloat16*>(a.y);
  g2.ldo = a.d;
  g2.x_res = static_cast<const __nv_bfloat16*>(a.x_res);
  g2.res_by_slot = false;
  g2.reverse_tiles = a.pair2;          // GEMM1 ran just before: its last rows are in L2
  if (a.res_by_slot && a.x_res != nullptr && a.mode2 == kModeCombine && a.pair2 &&
      a.x_disp != nullptr) {
    g2.x_res = static_cast<const __nv_bfloat16*>(a.x_disp);
    g2.res_by_slot = true;
  }
  g2.gate = a.gate;
  g2.comb_out = static_cast<__nv_bfloat16*>(a.out);
  if (a.mode2 == kModeCombineEp) {
    // expert parallelism: outputs go to each token's home rank (CTA pairs only)
    if (!a.pair2 || a.peer_out == nullptr || a.n_peers < 1 || a.n_peers > kEpMaxRanks)
      return cudaErrorInvalidValue;
    for (int i = 0; i < a.n_peers; ++i)
      g2.peer_out[i] = static_cast<__nv_bfloat16*>(a.peer_out[i]);
  }
  return a.pair2 ? run_gemm_pair<false>(ta2, ta2h, ta2q, tb2, to2, g2, a.num_sms, st)
                : run_gemm<false>(ta2, tb2, to2, g2, a.num_sms, st);
}

// ===================================================== fp32 CUDA cores

constexpr int kSB = 64, kSK = 16;

// grid (ceil(C / 64), ceil(n_out / 64), N); 256 threads, 4x4 outputs each.
__global__ void __launch_bounds__(256) ffn_simt_kernel(
    int mode, int64_t C, int n_out, int K, const int* __restrict__ counts,
    const int* __restrict__ slot_token, const float* __restrict__ a_src, bool a_gather,
    const float* __restrict__ w, float* __restrict__ out, const float* __restrict__ x_res,
    const float* __restrict__ gate) {
  __shared__ float As[kSK][kSB + 4];
  __shared__ float Bs[kSK][kSB + 4];
  const int e = blockIdx.z;
  const int64_t cnt = counts[e];
  const int64_t n_e = cnt < C ? cnt : C;
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * kSB;
  if (r0 >= n_e) return;
  const int c0 = blockIdx.y * kSB;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const float* wE = w + static_cast<int64_t>(e) * n_out * K;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += kSK) {
    for (int i = threadIdx.x; i < kSB * kSK; i += 256) {
      const int rr = i / kSK, kk = i % kSK;
      const int64_t r = r0 + rr;
      float v = 0.f;
      if (r < n_e && k0 + kk < K) {
        const int64_t src_row =
            a_gather ? static_cast<int64_t>(slot_token[static_cast<int64_t>(e) * C + r])
                     : static_cast<int64_t>(e) * C + r;
        v = a_src[src_row * K + k0 + kk];
      }
      As[kk][rr] = v;
      const int cc = c0 + rr;
      Bs[kk][rr] = (cc < n_out && k0 + kk < K) ? wE[static_cast<int64_t>(cc) * K + k0 + kk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kSK; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t r = r0 + ty * 4 + i;
    if (r >= n_e) continue;
    const int64_t slot = static_cast<int64_t>(e) * C + r;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int col = c0 + tx * 4 + j;
      if (col >= n_out) continue;
      if (mode == kModeHidden) {
        out[slot * n_out + col] = fmaxf(acc[i][j], 0.f);
      } else if (mode == kModeY) {
        out[slot * n_out + col] = acc[i][j];
      } else {
        const int tok = slot_token[slot];
        const float xr = x_res ? x_res[static_cast<int64_t>(tok) * n_out + col] : 0.f;
        out[static_cast<int64_t>(tok) * n_out + col] = fmaf(gate[tok], acc[i][j], xr);
      }
    }
  }
}

cudaError_t launch_expert_ffn_f32(const FfnArgs& a, cudaStream_t st) {
  const dim3 g1(static_cast<unsigned>((a.C + kSB - 1) / kSB),
                static_cast<unsigned>((a.F + kSB - 1) / kSB), static_cast<unsigned>(a.N));
  // token rows gathered through slot_token, or already dispatched
  const bool gather = a.x_disp == nullptr;
  ffn_simt_kernel<<<g1, 256, 0, st>>>(kModeHidden, a.C, a.F, a.d, a.counts, a.slot_token,
                                      static_cast<const float*>(gather ? a.x : a.x_disp), gather,
                                      static_cast<const float*>(a.w1),
                                      static_cast<float*>(a.hbuf), nullptr, nullptr);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || a.gemm1_only) return e;
  const dim3 g2(static_cast<unsigned>((a.C + kSB - 1) / kSB),
                static_cast<unsigned>((a.d + kSB - 1) / kSB), static_cast<unsigned>(a.N));
  float* out2 = a.mode2 == kModeCombine ? static_cast<float*>(a.out) : static_cast<float*>(a.y);
  ffn_simt_kernel<<<g2, 256, 0, st>>>(a.mode2, a.C, a.d, a.F, a.counts, a.slot_token,
                                      static_cast<const float*>(a.hbuf), false,
                                      static_cast<const float*>(a.w2), out2,
                                      static_cast<const float*>(a.x_res), a.gate);
  return cudaGetLastError();
}

}  // namespace smoe
