// Router: logits h = W_r . x (+ b), fp32 softmax, top-1 expert (lowest
// index on ties), gate p_idx, optional probabilities, per-tile column sums
// of the probabilities (for P_i of the balance loss).
//
// "Switch Transformers: scaling to trillion-parameter models": section
// "Switch Routing: From Top-k to k = 1" (router logits, gate equation, k = 1)
// and section "Making Sparse Training Stable" (router math in float32).
//
// Two implementations:
//  * router_simt_kernel: CUDA-core fp32 FMA; any N <= 1024, fp32 or bf16 x.
//  * router_tc_kernel: tcgen05 tensor cores for bf16 x.  bf16 values are
//    exact in fp32, and W_r is split into bf16 terms hi + mid + lo whose sum
//    is W_r exactly (8 + 8 + 8 significand bits cover fp32's 24), so every
//    product is exact and the tensor core only adds fp32 rounding in the
//    accumulation, like an FMA loop.  Accumulator in TMEM, one token per
//    TMEM lane; the softmax, argmax, probabilities, column sums and the
//    dispatch ranks of the tile run in the epilogue warps.
#include "kernels.cuh"

namespace smoe {

constexpr float kLog2e = 1.4426950408889634f;

// ================================================================ SIMT

constexpr int kSimtTok = 64;      // tokens per block (8 warps x 8)
constexpr int kSimtKC = 32;       // K chunk staged in shared memory

template <bool kBF16>
__global__ void __launch_bounds__(256) router_simt_kernel(
    int64_t T, int d, int N, const void* __restrict__ xv, const float* __restrict__ w_r,
    const float* __restrict__ b_r, float* __restrict__ logits, int* __restrict__ idx,
    float* __restrict__ gate, float* __restrict__ probs, float* __restrict__ psum) {
  extern __shared__ float sh[];
  float* Xs = sh;                              // [64][33]
  float* Ws = sh + kSimtTok * (kSimtKC + 1);   // [32][128]
  float* red = sh;                             // [8][N] (after the GEMM loops)
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int64_t tok0 = static_cast<int64_t>(blockIdx.x) * kSimtTok;

  for (int g0 = 0; g0 < N; g0 += 128) {
    float acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    for (int k0 = 0; k0 < d; k0 += kSimtKC) {
      for (int i = tid; i < kSimtTok * kSimtKC; i += 256) {
        const int r = i / kSimtKC, c = i % kSimtKC;
        const int64_t t = tok0 + r;
        float v = 0.f;
        if (t < T && k0 + c < d) {
          if (kBF16)
            v = __bfloat162float(static_cast<const __nv_bfloat16*>(xv)[t * d + k0 + c]);
          else
            v = static_cast<const float*>(xv)[t * d + k0 + c];
        }
        Xs[r * (kSimtKC + 1) + c] = v;
      }
      for (int i = tid; i < kSimtKC * 128; i += 256) {
        const int e = i / kSimtKC, c = i % kSimtKC;
        const int ge = g0 + e;
        Ws[c * 128 + e] = (ge < N && k0 + c < d) ? w_r[static_cast<int64_t>(ge) * d + k0 + c] : 0.f;
      }
      __syncthreads();
#pragma unroll 4
      for (int c = 0; c < kSimtKC; ++c) {
        float wv[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) wv[j] = Ws[c * 128 + lane + 32 * j];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float xs = Xs[(w * 8 + i) * (kSimtKC + 1) + c];
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(xs, wv[j], acc[i][j]);
        }
      }
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t t = tok0 + w * 8 + i;
      if (t >= T) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int e = g0 + lane + 32 * j;
        if (e < N) logits[t * N + e] = acc[i][j] + (b_r ? b_r[e] : 0.f);
      }
    }
  }
  __syncthreads();
  for (int i = tid; i < 8 * N; i += 256) red[i] = 0.f;
  __syncthreads();

  // softmax / argmax per token; lane owns experts lane + 32 m (same lanes
  // that wrote those logits above).
  for (int i = 0; i < 8; ++i) {
    const int64_t t = tok0 + w * 8 + i;
    if (t >= T) break;
    const float* row = logits + t * N;
    float best = -INFINITY;
    int best_e = 0x7fffffff;
    for (int e = lane; e < N; e += 32) {
      const float h = row[e];
      if (h > best) { best = h; best_e = e; }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, off);
      const int oe = __shfl_xor_sync(0xffffffffu, best_e, off);
      if (ob > best || (ob == best && oe < best_e)) { best = ob; best_e = oe; }
    }
    float s = 0.f;
    for (int e = lane; e < N; e += 32) s += exp2f((row[e] - best) * kLog2e);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    const float inv = 1.f / s;
    for (int e = lane; e < N; e += 32) {
      const float p = exp2f((row[e] - best) * kLog2e) * inv;
      if (probs) probs[t * N + e] = p;
      red[w * N + e] += p;
    }
    if (lane == 0) {
      idx[t] = best_e;
      gate[t] = inv;
    }
  }
  __syncthreads();
  if (psum) {
    for (int e = tid; e < N; e += 256) {
      float s = 0.f;
      for (int q = 0; q < 8; ++q) s += red[q * N + e];
      psum[static_cast<int64_t>(blockIdx.x) * N + e] = s;
    }
  }
}

cudaError_t launch_router_simt(int64_t T, int d, int N, bool bf16, const void* x,
                               const float* w_r, const float* b_r, float* logits,
                               RouterOut o, int* nparts_out, cudaStream_t st) {
  const int blocks = static_cast<int>((T + kSimtTok - 1) / kSimtTok);
  *nparts_out = blocks;
  size_t sm = sizeof(float) * (kSimtTok * (kSimtKC + 1) + kSimtKC * 128);
  if (sizeof(float) * 8 * N > sm) sm = sizeof(float) * 8 * N;
  if (bf16)
    router_simt_kernel<true><<<blocks, 256, sm, st>>>(T, d, N, x, w_r, b_r, logits, o.idx,
                                                     o.gate, o.probs, o.psum);
  else
    router_simt_kernel<false><<<blocks, 256, sm, st>>>(T, d, N, x, w_r, b_r, logits, o.idx,
                                                      o.gate, o.probs, o.psum);
  return cudaGetLastError();
}

// ======================================================== tensor cores

__global__ void wsplit_kernel(int N, int N_pad, int d, int terms,
                              const float* __restrict__ w_r, __nv_bfloat16* __restrict__ out) {
  const int64_t n = static_cast<int64_t>(N_pad) * d;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int e = static_cast<int>(i / d);
    const float w = e < N ? w_r[i] : 0.f;
    const __nv_bfloat16 hi = __float2bfloat16_rn(w);
    const float r1 = w - __bfloat162float(hi);           // exact
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(mid);          // exact
    out[i] = hi;
    out[n + i] = mid;
    if (terms == 3) out[2 * n + i] = __float2bfloat16_rn(r2);   // exact: r2 has <= 8 bits
  }
}

struct RouterTcParams {
  int64_t T;
  int d, N, N_pad, acc_stride, terms, stages, ntiles;
  uint32_t stage_bytes, tmem_cols;
  const float* b_r;
  RouterOut o;
  DevErr* err;
  long long spin;
};

constexpr int kRouterThreads = 192;   // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue

__device__ __forceinline__ void transpose_reduce32(float (&v)[32], int lane) {
  // After this, lane j holds the sum over the warp's lanes of v[j].
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < off; ++i) {
      const float send = upper ? v[i] : v[i + off];
      const float keep = upper ? v[i + off] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
}

__global__ void __launch_bounds__(kRouterThreads, 1) router_tc_kernel(
    const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
    RouterTcParams prm) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const int S = prm.stages;
  uint8_t* tail = smem + static_cast<size_t>(S) * prm.stage_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(tail);
  uint64_t* empty = full + 8;
  uint64_t* tfull = empty + 8;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* epi_abort = abort_flag + 1;
  const int NS = prm.acc_stride;                       // N_pad rounded up to 32
  float* bias_s = reinterpret_cast<float*>(tail + 256);  // [NS]
  float* red = bias_s + NS;                              // [4][NS]
  int* cnt = reinterpret_cast<int*>(red + 4 * NS);       // [4][N_pad]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = prm.N, N_pad = prm.N_pad;
  const int kblocks = prm.d / 64;
  const long long lim = prm.spin;
  const uint32_t a_bytes = 128 * 128;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    *epi_abort = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  for (int i = threadIdx.x; i < NS; i += blockDim.x)
    bias_s[i] = (prm.b_r != nullptr && i < N) ? prm.b_r[i] : 0.f;
  if (warp == 1) {
    tmem_alloc(tmem_holder, prm.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmap_x);
      tma_prefetch_desc(&tmap_w);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_phase = 0;
      for (int tile = blockIdx.x; tile < prm.ntiles && !*abort_flag; tile += gridDim.x) {
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, lim)) {
            report_error(prm.err, SWITCH_ERR_TIMEOUT, kWhereRouterProducer, tile);
            *abort_flag = 1;
            break;
          }
          uint8_t* sa = smem + static_cast<size_t>(stage) * prm.stage_bytes;
          uint8_t* sb = sa + a_bytes;
          mbar_arrive_expect_tx(&full[stage], prm.stage_bytes);
          tma_load_2d(sa, &tmap_x, &full[stage], kb * 64, tile * 128);
          for (int p = 0; p < prm.terms; ++p)
            tma_load_2d(sb + static_cast<size_t>(p) * N_pad * 128, &tmap_w, &full[stage],
                        kb * 64, p * N_pad);
          issued_mask |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
      }
      // Never leave with copies in flight into this CTA's shared memory.
      for (int s = 0; s < S; ++s)
        if (((issued_mask >> s) & 1u) &&
            !mbar_wait(&full[s], (issued_phase >> s) & 1u, kDefaultSpinCycles))
          report_error(prm.err, SWITCH_ERR_TIMEOUT, kWhereDrain, s);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, N_pad);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool any = false;
      for (int tile = blockIdx.x; tile < prm.ntiles && !*abort_flag; tile += gridDim.x) {
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, lim)) {
          report_error(prm.err, SWITCH_ERR_TIMEOUT, kWhereRouterMma, tile);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * prm.acc_stride);
        bool ok = true;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&full[stage], phase, lim)) {
            report_error(prm.err, SWITCH_ERR_TIMEOUT, kWhereRouterMma, tile);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + static_cast<size_t>(stage) * prm.stage_bytes);
          const uint32_t sb = sa + a_bytes;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t ad = sw128_kmajor_desc(sa + k * 32);
            for (int p = 0; p < prm.terms; ++p) {
              const uint64_t bd =
                  sw128_kmajor_desc(sb + static_cast<uint32_t>(p * N_pad * 128) + k * 32);
              umma_bf16(d_tmem, ad, bd, idesc, (kb | k | p) != 0 ? 1u : 0u);
            }
          }
          any = true;
          umma_commit(&empty[stage]);
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (any && *abort_flag) {
        // Let every issued MMA finish before TMEM is released.
        umma_commit(drain);
        if (!mbar_wait(drain, 0, kDefaultSpinCycles))
          report_error(prm.err, SWITCH_ERR_TIMEOUT, kWhereDrain, -1);
      }
    }
  } else {
    // ------------------------------------------------------- epilogue
    const int q = warp & 3;                 // TMEM lane quarter of this warp
    const int row = q * 32 + lane;
    const int et = threadIdx.x - 64;        // 0..127
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < prm.ntiles; tile += gridDim.x) {
      const bool ok = mbar_wait(&tfull[acc], acc_phase, lim);
      if (!ok) *epi_abort = 1;
      for (int i = et; i < 4 * N_pad; i += 128) cnt[i] = 0;
      named_bar_sync(1, 128);
      if (*epi_abort || *abort_flag) {
        if (et == 0) {
          report_error(prm.err, SWITCH_ERR_TIMEOUT, kWhereRouterEpilogue, tile);
          *abort_flag = 1;
        }
        break;
      }
      tc_fence_after();
      const int64_t t = static_cast<int64_t>(tile) * 128 + row;
      const bool valid = t < prm.T;
      const uint32_t taddr =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * prm.acc_stride);
      float v[32];
      // pass 1: max and argmax (lowest index on ties)
      float m = -INFINITY;
      int best = 0;
      for (int c = 0; c < N_pad; c += 32) {
        tmem_ld32(taddr + c, v);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int e = c + j;
          const float h = v[j] + bias_s[e];
          if (e < N && h > m) { m = h; best = e; }
        }
      }
      // pass 2: sum of exponentials
      float s = 0.f;
      for (int c = 0; c < N_pad; c += 32) {
        tmem_ld32(taddr + c, v);
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (c + j < N) s += exp2f((v[j] + bias_s[c + j] - m) * kLog2e);
      }
      const float inv = 1.f / s;
      // pass 3: probabilities, their column sums over the tile
      for (int c = 0; c < N_pad; c += 32) {
        tmem_ld32(taddr + c, v);
#pragma unroll
        for (int j = 0; j < 32; ++j)
          v[j] = (valid && c + j < N) ? exp2f((v[j] + bias_s[c + j] - m) * kLog2e) * inv : 0.f;
        if (valid && prm.o.probs != nullptr) {
          float4* dst = reinterpret_cast<float4*>(prm.o.probs + t * N + c);
          if (c + 32 <= N && (N % 4) == 0) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
              dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
          } else {
            for (int j = 0; j < 32 && c + j < N; ++j) prm.o.probs[t * N + c + j] = v[j];
          }
        }
        transpose_reduce32(v, lane);
        red[q * NS + c + lane] = v[0];
      }
      // accumulator consumed: hand it back to the MMA warp
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;

      if (valid) {
        prm.o.idx[t] = best;
        prm.o.gate[t] = inv;
      }
      // rank within the tile, token order (quarter q holds rows 32q..32q+31)
      const int e_key = valid ? best : -1;
      const unsigned peers = __match_any_sync(0xffffffffu, e_key);
      const int rank_w = __popc(peers & ((1u << lane) - 1u));
      if (valid && rank_w == 0) cnt[q * N_pad + best] = __popc(peers);
      named_bar_sync(1, 128);
      if (valid && prm.o.local_rank != nullptr) {
        int r = rank_w;
        for (int qq = 0; qq < q; ++qq) r += cnt[qq * N_pad + best];
        prm.o.local_rank[t] = r;
      }
      for (int e = et; e < N; e += 128) {
        if (prm.o.psum != nullptr)
          prm.o.psum[static_cast<int64_t>(tile) * N + e] =
              ((red[e] + red[NS + e]) + red[2 * NS + e]) + red[3 * NS + e];
        if (prm.o.hist != nullptr)
          prm.o.hist[static_cast<int64_t>(e) * prm.ntiles + tile] =
              cnt[e] + cnt[N_pad + e] + cnt[2 * N_pad + e] + cnt[3 * N_pad + e];
      }
      named_bar_sync(1, 128);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, prm.tmem_cols);
}

// ------------------------------------------------------------------ host

typedef CUresult (*PFN_encodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                    const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                    const cuuint32_t*, CUtensorMapInterleave,
                                    CUtensorMapSwizzle, CUtensorMapL2promotion,
                                    CUtensorMapFloatOOBfill);

PFN_encodeTiled get_encode_fn();   // defined in expert_ffn.cu

bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                       uint32_t box_inner, uint32_t box_outer);   // expert_ffn.cu

static int router_n_pad(int N) { return (N + 15) / 16 * 16; }

bool router_tc_supported(int N, int d, int terms) {
  const int n_pad = router_n_pad(N);
  return (terms == 2 || terms == 3) && n_pad <= 256 && d % 64 == 0 && d > 0;
}

cudaError_t launch_router_tc(int64_t T, int d, int N, int terms, const void* x,
                             const float* w_r, const float* b_r, void* wsplit, RouterOut o,
                             int ntiles, DevErr* err, long long spin, int num_sms,
                             cudaStream_t st) {
  const int N_pad = router_n_pad(N);
  {
    const int64_t n = static_cast<int64_t>(N_pad) * d;
    int blocks = static_cast<int>((n + 255) / 256);
    if (blocks > 1024) blocks = 1024;
    wsplit_kernel<<<blocks, 256, 0, st>>>(N, N_pad, d, terms, w_r,
                                          static_cast<__nv_bfloat16*>(wsplit));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  CUtensorMap tx, tw;
  if (!make_tmap_bf16_2d(&tx, x, static_cast<uint64_t>(d), static_cast<uint64_t>(T), 64, 128))
    return cudaErrorInvalidValue;
  if (!make_tmap_bf16_2d(&tw, wsplit, static_cast<uint64_t>(d),
                         static_cast<uint64_t>(terms) * N_pad, 64, static_cast<uint32_t>(N_pad)))
    return cudaErrorInvalidValue;

  RouterTcParams p;
  p.T = T;
  p.d = d;
  p.N = N;
  p.N_pad = N_pad;
  p.terms = terms;
  p.ntiles = ntiles;
  p.stage_bytes = 128u * 128u + static_cast<uint32_t>(terms) * N_pad * 128u;
  const int ns = (N_pad + 31) / 32 * 32;
  const size_t tail_bytes = 256 + sizeof(float) * ns * 5 + sizeof(int) * N_pad * 4;
  const size_t budget = 227 * 1024 - 1024 - tail_bytes;
  int stages = static_cast<int>(budget / p.stage_bytes);
  if (stages > 8) stages = 8;
  if (stages < 2) return cudaErrorInvalidConfiguration;
  p.stages = stages;
  // Accumulators start 32-column aligned so that the epilogue's 32-column
  // TMEM loads stay inside the allocation.
  p.acc_stride = ns;
  uint32_t cols = 32;
  while (cols < static_cast<uint32_t>(2 * p.acc_stride)) cols <<= 1;
  p.tmem_cols = cols;
  p.b_r = b_r;
  p.o = o;
  p.err = err;
  p.spin = spin;
  const size_t smem = 1024 + static_cast<size_t>(stages) * p.stage_bytes + tail_bytes;
  cudaError_t e = cudaFuncSetAttribute(router_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int grid = ntiles < num_sms ? ntiles : num_sms;
  router_tc_kernel<<<grid, kRouterThreads, smem, st>>>(tx, tw, p);
  return cudaGetLastError();
}

}  // namespace smoe
