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
//   * dX: dx[token] = dout[token] (residual) + router term + dX row.
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
    r.kblocks = p.K / kBK;
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

// Weight gradient rows: out[e * M_out + r, n * 256 + ...] = bf16(acc).
__device__ __forceinline__ void epi_store(const BwdParams& p, const BTile& t, uint32_t taddr,
                                          int q, int lane) {
  const int r = t.m * kBM + q * 32 + lane;
  const bool rv = r < p.M_out;
  const int cols = p.n_out - t.n * kBN < kBN ? p.n_out - t.n * kBN : kBN;
  __nv_bfloat16* orow = p.out + (static_cast<int64_t>(t.e) * p.M_out + r) * p.n_out + t.n * kBN;
  for (int c = 0; c < cols / 32; ++c) {
    uint32_t v[32];
    if (t.kblocks > 0) {
      tmem_ld32_issue(taddr + static_cast<uint32_t>(c * 32), v);
      tmem_ld_wait(v);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = 0u;
    }
    if (rv) {
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
__device__ __forceinline__ void epi_dh(const BwdParams& p, const BTile& t, uint32_t taddr,
                                       int q, int lane) {
  const int64_t r_in = static_cast<int64_t>(t.m) * kBM + q * 32 + lane;
  const int64_t cnt = p.counts[t.e];
  const int64_t ne = cnt < p.C ? cnt : p.C;
  const bool in_cap = r_in < p.C;
  const bool kept = r_in < ne;
  const int64_t s = static_cast<int64_t>(t.e) * p.C + r_in;
  const int cols = p.n_out - t.n * kBN < kBN ? p.n_out - t.n * kBN : kBN;
  const int64_t off = s * p.n_out + t.n * kBN;
  float dot = 0.f;
  for (int c = 0; c < cols / 32; ++c) {
    uint32_t v[32];
    tmem_ld32_issue(taddr + static_cast<uint32_t>(c * 32), v);
    tmem_ld_wait(v);
    if (in_cap) {
      uint4 hv[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) hv[k] = ld_u4(p.h + off + c * 32 + 8 * k);
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
  }
  if (kept) p.dgp[s * p.ntiles_n + t.n] = dot;
}

// dX tile: rows are slots; kept slots write their token's input gradient
// dx[t] = (residual ? dout[t] : 0) + dxr[t] + acc, rounded once.
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
        const float4 r0 = __ldg(reinterpret_cast<const float4*>(p.dxr + o8));
        const float4 r1 = __ldg(reinterpret_cast<const float4*>(p.dxr + o8 + 4));
        float a[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
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

}  // namespace

template <int kSched, int kEpi>
__global__ void __launch_bounds__(kBwdThreads, 1) bwd_gemm_kernel(
    const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
    BwdParams p) {
  constexpr bool kAMN = kSched == kSchedWeight;     // rows: A K-major; weight: A MN-major
  const int total = kSched == kSchedRows ? p.mtile_start[p.N] * p.ntiles_n
                                         : p.N * p.ntiles_m * p.ntiles_n;
  if (static_cast<int>(blockIdx.x) >= total) return;    // uniform for the block

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* tail = smem + kBwdStages * kBwdStageBytes;
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
          if (kSched == kSchedRows) {
            // A: 128 slot rows x 64 K, K-major; B: MN-major boxes of the
            // expert's weight rows kb*64.. (64 K rows x 64 output columns)
            tma_load_2d(sa, &tmap_a, &full[stage], kb * kBK,
                        static_cast<int>(static_cast<int64_t>(t.e) * p.C + t.m * kBM));
#pragma unroll
            for (int j = 0; j < 4; ++j)
              tma_load_2d(sb + j * kBox, &tmap_b, &full[stage], t.n * kBN + 64 * j,
                          t.e * p.b_rows + kb * kBK);
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
    int acc = 0;
    uint32_t acc_phase = 0;
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
      if (kEpi == kEpiStore) epi_store(p, t, taddr, q, lane);
      else if (kEpi == kEpiDH) epi_dh(p, t, taddr, q, lane);
      else epi_dx(p, t, taddr, q, lane);
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

// ------------------------------------------------------------------- host

// 3-D bf16 tensor [outer][mid][inner] (inner contiguous), 128-byte swizzle,
// box box_inner x box_mid x 1; out-of-range elements read as zero.
static bool make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t mid,
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
static cudaError_t run_bwd(const CUtensorMap& ta, const CUtensorMap& tb, const BwdParams& p,
                           int num_sms, cudaStream_t st) {
  const size_t smem = 1024 + kBwdStages * kBwdStageBytes + 128 + sizeof(int) * (p.N + 1);
  static size_t smem_set[64] = {};
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(&bwd_gemm_kernel<kSched, kEpi>),
                                    smem, smem_set);
  if (e != cudaSuccess) return e;
  bwd_gemm_kernel<kSched, kEpi><<<num_sms, kBwdThreads, smem, st>>>(ta, tb, p);
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
  CUtensorMap ta, tb;
  bool ok = make_tmap_bf16_2d(&ta, a.dys, a.d, slots, kBK, kBM);
  ok = ok && make_tmap_bf16_2d(&tb, a.w2, a.F, static_cast<uint64_t>(a.N) * a.d, 64, 64);
  if (!ok) return cudaErrorInvalidValue;
  BwdParams p = base_params(a);
  p.K = a.d;
  p.n_out = a.F;
  p.ntiles_n = (a.F + kBN - 1) / kBN;
  p.b_rows = a.d;
  p.h = static_cast<const __nv_bfloat16*>(a.hbuf);
  p.out = static_cast<__nv_bfloat16*>(a.da);
  p.dgp = a.dgp;
  return run_bwd<kSchedRows, kEpiDH>(ta, tb, p, a.num_sms, st);
}

cudaError_t launch_bwd_dw(const BwdFfnArgs& a, cudaStream_t st) {
  CUtensorMap ta2, tb2, ta1, tb1;
  const uint64_t C = static_cast<uint64_t>(a.C), N = static_cast<uint64_t>(a.N);
  bool ok = make_tmap_bf16_3d(&ta2, a.dys, a.d, C, N, 64, kBK);
  ok = ok && make_tmap_bf16_3d(&tb2, a.hbuf, a.F, C, N, 64, kBK);
  ok = ok && make_tmap_bf16_3d(&ta1, a.da, a.F, C, N, 64, kBK);
  ok = ok && make_tmap_bf16_3d(&tb1, a.x_disp, a.d, C, N, 64, kBK);
  if (!ok) return cudaErrorInvalidValue;
  // dW2_e [d, F] = dY_e^T H_e
  BwdParams p2 = base_params(a);
  p2.M_out = a.d;
  p2.n_out = a.F;
  p2.ntiles_m = (a.d + kBM - 1) / kBM;
  p2.ntiles_n = (a.F + kBN - 1) / kBN;
  p2.out = static_cast<__nv_bfloat16*>(a.dw2);
  cudaError_t e = run_bwd<kSchedWeight, kEpiStore>(ta2, tb2, p2, a.num_sms, st);
  if (e != cudaSuccess) return e;
  // dW1_e [F, d] = dA_e^T X_e
  BwdParams p1 = base_params(a);
  p1.M_out = a.F;
  p1.n_out = a.d;
  p1.ntiles_m = (a.F + kBM - 1) / kBM;
  p1.ntiles_n = (a.d + kBN - 1) / kBN;
  p1.out = static_cast<__nv_bfloat16*>(a.dw1);
  return run_bwd<kSchedWeight, kEpiStore>(ta1, tb1, p1, a.num_sms, st);
}

cudaError_t launch_bwd_dx(const BwdFfnArgs& a, cudaStream_t st) {
  const uint64_t slots = static_cast<uint64_t>(a.N) * static_cast<uint64_t>(a.C);
  CUtensorMap ta, tb;
  bool ok = make_tmap_bf16_2d(&ta, a.da, a.F, slots, kBK, kBM);
  ok = ok && make_tmap_bf16_2d(&tb, a.w1, a.d, static_cast<uint64_t>(a.N) * a.F, 64, 64);
  if (!ok) return cudaErrorInvalidValue;
  BwdParams p = base_params(a);
  p.K = a.F;
  p.n_out = a.d;
  p.ntiles_n = (a.d + kBN - 1) / kBN;
  p.b_rows = a.F;
  p.dout = static_cast<const __nv_bfloat16*>(a.dout);
  p.dxr = a.dxr;
  p.dx = static_cast<__nv_bfloat16*>(a.dx);
  p.residual = a.residual ? 1 : 0;
  return run_bwd<kSchedRows, kEpiDX>(ta, tb, p, a.num_sms, st);
}

}  // namespace smoe
