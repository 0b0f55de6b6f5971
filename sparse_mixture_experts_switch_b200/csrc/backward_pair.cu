// Backward dX GEMM of the expert FFNs on CTA pairs with the operands swapped
// ("Switch Transformers: scaling to trillion-parameter models", section
// "The Core Idea": the input gradient of E_e(x) = relu(x W1_e^T) W2_e^T is
// dA W1_e; section "Switch Routing": the router's gradient dh reaches x
// through h = W_r x, adding dh W_r; the residual branch adds dout).
//
// The accumulator holds the transposed tile, input features x slots:
//
//   D[k, j] = sum_f W1[e][f, k] dA[slot j, f]  +  sum_i W_r[i, k] dh[slot j, i]
//
// the router term as three extra bf16 split terms of the same accumulation
// (W_r hi . dh hi, W_r hi . dh lo, W_r lo . dh hi; dh's planes are stored per
// kept slot, zero where the slot does not carry the token's router term).
// A pair tile is 256 input features x up to 256 of one expert's kept slots;
// the MMA's N is the slot count rounded up to 16, so an expert's ragged last
// tile wastes at most 15 columns.  CTA r of the pair holds features
// f0 + 128 r .. + 127 of W1 (stored [d_ff, d]: the A operand is MN-major, two
// 64 x 64 TMA boxes per K step; W_r's planes likewise) and slot rows
// r * N/2 .. of dA (K-major, one box; dh's planes likewise); the leader
// issues tcgen05.mma.cta_group::2 (M = 256, N = 16..256, K = 16) and each
// CTA's TMEM receives its 128 features x N slots.  Every SM streams 32 KB per
// 64-deep K step, and each W1 tile is read once per 256 slots.  No copy is
// multicast.
//
// Epilogue (one warp per 32 features): each 32-slot chunk is transposed
// through shared memory so that a lane owns 8 features of one slot, then
//   top-1: dx[token] = (residual ? dout[token] : 0) + acc, one bf16 rounding,
//          16-byte accesses (the next tile's dout rows are prefetched into L2
//          while this tile's main loop runs);
//   top-2: the fp32 row is stored at the slot (dxs), to be added per token.
#include <cstring>

#include "backward.cuh"
#include "gemm_pair.cuh"

namespace smoe {

namespace {

constexpr uint32_t kBoxBytes = 64 * 64 * 2;                 // one 64 x 64 bf16 box
constexpr int kDxThreads = 192;                             // w0 TMA, w1 MMA, w2-5 epilogue
constexpr uint32_t kDxStageBytes = 2 * kBoxBytes + kPairTokBytes;   // W half + slot rows

struct DxPairParams {
  GemmParams g;             // N, n_out = d, K = d_ff, ntiles_n, C, counts, mtile_start,
                            // slot_token, err, spin
  int kx_blocks;            // router term: K blocks per split term (Np / 64)
  const __nv_bfloat16* dout;
  __nv_bfloat16* dx;
  float* dxs;               // top-2: [N*C, d] fp32 rows per slot (dx untouched)
  int residual;
};

// The token rows of dout that tile t's epilogue will read for the warp's 32
// features, into L2 (lane j takes slots j, j + 32, ...).
__device__ __forceinline__ void prefetch_dout(const DxPairParams& P, const PairTile& t, int fb,
                                              int lane) {
  if (!P.residual || P.dxs != nullptr || fb >= P.g.n_out) return;
  const int64_t row0 = static_cast<int64_t>(t.e) * P.g.C + t.t0;
  for (int j = lane; j < t.nv; j += 32)
    prefetch_l2(P.dout + static_cast<int64_t>(P.g.slot_token[row0 + j]) * P.g.n_out + fb);
}

}  // namespace

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kDxThreads, 1)
    bwd_dx_pair_kernel(const __grid_constant__ CUtensorMap tmap_w1,
                       const __grid_constant__ CUtensorMap tmap_da,
                       const __grid_constant__ CUtensorMap tmap_wr,
                       const __grid_constant__ CUtensorMap tmap_dh, DxPairParams P) {
  const GemmParams& p = P.g;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* stage_out = smem + kPairStages * kDxStageBytes;           // [4][4 KB], 1024-aligned
  uint8_t* tail = stage_out + 4 * kStageOutBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(tail);   // leader: TMA bytes of both CTAs
  uint64_t* empty = full + kPairStages;                  // local: stage free (MMA done)
  uint64_t* tfull = empty + kPairStages;                 // local: accumulator ready
  uint64_t* tempty = tfull + 2;                          // leader: accumulator drained
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tail + 192);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tail + 196);
  int* mts = reinterpret_cast<int*>(tail + 256);                        // [N + 1]
  int* pts = mts + (p.N + 1);                                           // [N + 1]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cid = static_cast<int>(cluster_id_x());
  const int ncl = static_cast<int>(cluster_count_x());
  const long long lim = p.spin;
  const int kmain = p.K / kBK;
  const int kblocks = kmain + 3 * P.kx_blocks;

  for (int i = threadIdx.x; i <= p.N; i += blockDim.x) mts[i] = p.mtile_start[i];
  __syncthreads();
  if (warp == 0) pair_prefix_warp(p.N, mts, pts);
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
      tma_prefetch_desc(&tmap_w1);
      tma_prefetch_desc(&tmap_da);
      tma_prefetch_desc(&tmap_wr);
      tma_prefetch_desc(&tmap_dh);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_phase = 0;
      for (int tile = cid; tile < total && !*abort_flag; tile += ncl) {
        const PairTile t = pair_tile(p, pts, tile);
        const int tok_row = static_cast<int>(static_cast<int64_t>(t.e) * p.C + t.t0 +
                                             static_cast<int>(rank) * (t.nmma >> 1));
        const int f_col = t.f0 + static_cast<int>(rank) * 128;
        bool ok = true;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, lim)) {
            report_error(p.err, SWITCH_ERR_TIMEOUT, kWhereGemmProducer, tile);
            *abort_flag = 1;
            ok = false;
            break;
          }
          uint8_t* sw = smem + stage * kDxStageBytes;
          uint8_t* stok = sw + 2 * kBoxBytes;
          const uint32_t bar = full_lead + 8u * stage;
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * kDxStageBytes);
          if (kb < kmain) {
            // W1 viewed as [N*d_ff rows, d columns]: rows e*d_ff + kb*64 ..,
            // this CTA's feature columns (MN-major boxes); dA slot rows
#pragma unroll
            for (int j = 0; j < 2; ++j)
              tma_load_2d_pair(sw + j * kBoxBytes, &tmap_w1, bar, f_col + 64 * j,
                               t.e * p.K + kb * kBK);
            tma_load_2d_pair(stok, &tmap_da, bar, kb * kBK, tok_row);
          } else {
            // router term: W_r plane (lo for the third term) x dh plane (lo
            // for the second term)
            const int x = kb - kmain;
            const int term = x / P.kx_blocks;
            const int kk = x - term * P.kx_blocks;
#pragma unroll
            for (int j = 0; j < 2; ++j)
              tma_load_3d_pair(sw + j * kBoxBytes, &tmap_wr, bar, f_col + 64 * j, kk * kBK,
                               term == 2 ? 1 : 0);
            tma_load_3d_pair(stok, &tmap_dh, bar, kk * kBK, tok_row, term == 1 ? 1 : 0);
          }
          issued_mask |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == kPairStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
      }
      // both CTAs' TMA bytes complete on the leader's barriers, which the
      // leader drains before the final cluster barrier
      if (leader)
        for (int s = 0; s < kPairStages; ++s)
          if (((issued_mask >> s) & 1u) &&
              !mbar_wait_cluster(&full[s], (issued_phase >> s) & 1u, kDefaultSpinCycles))
            report_error(p.err, SWITCH_ERR_TIMEOUT, kWhereDrain, s);
    }
  } else if (warp == 1) {
    // ------------------------------------------------- MMA issuer (leader)
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool any = false;
      for (int tile = cid; tile < total && !*abort_flag; tile += ncl) {
        const uint32_t idesc =
            idesc_bf16_f32_major(2 * kBM, pair_tile(p, pts, tile).nmma, true, false);
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
          const uint32_t sw = smem_u32(smem + stage * kDxStageBytes);
          const uint32_t stok = sw + 2 * kBoxBytes;
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)
            umma_bf16_pair(d_tmem, sw128_mnmajor_desc(sw + k * 2048, kBoxBytes),
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
    }
  } else {
    // ------------------------------------------------------- epilogue warps
    const int q = warp & 3;                 // TMEM lane quarter: features fq .. fq + 31
    const uint32_t stg = smem_u32(stage_out + q * kStageOutBytes);
    const int fq = static_cast<int>(rank) * 128 + q * 32;
    const int qq = lane & 3;                // 8-feature group of this lane
    const int rr0 = lane >> 2;              // slot row within an 8-row pass
    int acc = 0;
    uint32_t acc_phase = 0;
    {
      const PairTile t0 = pair_tile(p, pts, cid);
      prefetch_dout(P, t0, t0.f0 + fq, lane);
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
      if (tile + ncl < total) {
        const PairTile tn = pair_tile(p, pts, tile + ncl);
        prefetch_dout(P, tn, tn.f0 + fq, lane);
      }
      const int fb = t.f0 + fq;
      const int64_t row0 = static_cast<int64_t>(t.e) * p.C + t.t0;
      const int nch = (t.nv + 31) >> 5;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc * kBN);
      if (fb < p.n_out) {                     // warp-uniform: features of this warp exist
        for (int c = 0; c < nch; ++c) {
          uint32_t u[32];
          tmem_ld32_issue(taddr + static_cast<uint32_t>(c * 32), u);
          const int jl = c * 32 + lane;
          const int tokc = (P.dxs == nullptr && jl < t.nv) ? p.slot_token[row0 + jl] : -1;
          tmem_ld_wait(u);
          // transpose: element (slot j, feature lane) at row j, 16-byte chunk
          // (lane / 4) ^ (j % 8) of a 128-byte row
#pragma unroll
          for (int j = 0; j < 32; ++j)
            st_shared_f32(stg + j * 128 + ((((lane >> 2) ^ j) & 7) << 4) + (lane & 3) * 4,
                          __uint_as_float(u[j]));
          __syncwarp();
          int tk[4];
          uint4 res[4];
#pragma unroll
          for (int pass = 0; pass < 4; ++pass) {
            tk[pass] = __shfl_sync(0xffffffffu, tokc, pass * 8 + rr0);
            res[pass] = make_uint4(0, 0, 0, 0);
            if (tk[pass] >= 0 && P.residual)
              res[pass] = __ldg(reinterpret_cast<const uint4*>(
                  P.dout + static_cast<int64_t>(tk[pass]) * p.n_out + fb + qq * 8));
          }
#pragma unroll
          for (int pass = 0; pass < 4; ++pass) {
            const int rr = pass * 8 + rr0;
            const int j = c * 32 + rr;
            if (j >= t.nv) continue;
            const float4 a = ld_shared_v4(stg + rr * 128 + (((2 * qq) ^ (rr & 7)) << 4));
            const float4 b = ld_shared_v4(stg + rr * 128 + (((2 * qq + 1) ^ (rr & 7)) << 4));
            if (P.dxs != nullptr) {
              float4* dst = reinterpret_cast<float4*>(P.dxs + (row0 + j) * p.n_out + fb + qq * 8);
              dst[0] = a;
              dst[1] = b;
            } else {
              const uint4 r = res[pass];
              uint4 o;
              o.x = pack_bf16x2(bf16_lo(r.x) + a.x, bf16_hi(r.x) + a.y);
              o.y = pack_bf16x2(bf16_lo(r.y) + a.z, bf16_hi(r.y) + a.w);
              o.z = pack_bf16x2(bf16_lo(r.z) + b.x, bf16_hi(r.z) + b.y);
              o.w = pack_bf16x2(bf16_lo(r.w) + b.z, bf16_hi(r.w) + b.w);
              *reinterpret_cast<uint4*>(P.dx + static_cast<int64_t>(tk[pass]) * p.n_out + fb +
                                        qq * 8) = o;
            }
          }
          __syncwarp();                       // the buffer is rewritten by the next chunk
        }
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
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();                          // no CTA leaves while its peer may still signal it
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, kTmemCols);
}

size_t bwd_dx_pair_smem_bytes(int N) {
  return 1024 + kPairStages * kDxStageBytes + 4 * kStageOutBytes + 256 +
         2 * sizeof(int) * (N + 1);
}

cudaError_t launch_bwd_dx_pair(const BwdFfnArgs& a, cudaStream_t st) {
  const uint64_t slots = static_cast<uint64_t>(a.N) * static_cast<uint64_t>(a.C);
  CUtensorMap tw1, tda, twr, tdh;
  bool ok = make_tmap_bf16_2d(&tw1, a.w1, a.d, static_cast<uint64_t>(a.N) * a.F, 64, 64);
  ok = ok && make_tmap_bf16_2d(&tda, a.da, a.F, slots, kBK, 128);
  // router term: W_r planes [2][Np][d] (MN-major 64 x 64 boxes; rows N..Np-1
  // zero) and dh planes per slot [2][slots][Np] (K-major, 128-row boxes)
  ok = ok && make_tmap_bf16_3d(&twr, a.wrp, a.d, a.n_pad, 2, 64, kBK);
  ok = ok && make_tmap_bf16_3d(&tdh, a.dhs, a.n_pad, slots, 2, kBK, 128);
  if (!ok) return cudaErrorInvalidValue;
  DxPairParams P{};
  P.g.N = a.N;
  P.g.n_out = a.d;
  P.g.K = a.F;
  P.g.ntiles_n = (a.d + kBN - 1) / kBN;
  P.g.C = a.C;
  P.g.counts = a.counts;
  P.g.mtile_start = a.mtile_start;
  P.g.slot_token = a.slot_token;
  P.g.err = a.err;
  P.g.spin = a.spin;
  P.kx_blocks = a.n_pad / kBK;
  P.dout = static_cast<const __nv_bfloat16*>(a.dout);
  P.dx = static_cast<__nv_bfloat16*>(a.dx);
  P.dxs = a.dxs;
  P.residual = a.residual ? 1 : 0;
  const size_t smem = bwd_dx_pair_smem_bytes(a.N);
  static size_t smem_set[64] = {};
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(&bwd_dx_pair_kernel), smem,
                                    smem_set);
  if (e != cudaSuccess) return e;
  const int grid = (a.num_sms / 2) * 2;
  bwd_dx_pair_kernel<<<grid, kDxThreads, smem, st>>>(tw1, tda, twr, tdh, P);
  return cudaGetLastError();
}

}  // namespace smoe
