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

// 2^x on the special-function unit (one instruction).  Results below the
// smallest normal float (2^-126) flush to zero: a probability that small is
// reported as 0.
__device__ __forceinline__ float exp2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ================================================================ SIMT

constexpr int kSimtTok = 64;      // tokens per block (8 warps x 8)
constexpr int kSimtKC = 32;       // K chunk staged in shared memory

template <bool kBF16>
__global__ void __launch_bounds__(256) router_simt_kernel(
    int64_t T, int d, int N, const void* __restrict__ xv, const float* __restrict__ w_r,
    const float* __restrict__ b_r, float* __restrict__ logits, int* __restrict__ idx,
    float* __restrict__ gate, float* __restrict__ probs, float* __restrict__ psum,
    int* __restrict__ idx2, float* __restrict__ gate2) {
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
    // the two largest logits (value, index), lowest index first on ties:
    // per lane over its experts in increasing order, then merged across lanes
    float best = -INFINITY, sec = -INFINITY;
    int best_e = 0x7fffffff, sec_e = 0x7fffffff;
    for (int e = lane; e < N; e += 32) {
      const float h = row[e];
      if (h > best) { sec = best; sec_e = best_e; best = h; best_e = e; }
      else if (h > sec) { sec = h; sec_e = e; }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, off);
      const int oe = __shfl_xor_sync(0xffffffffu, best_e, off);
      const float os = __shfl_xor_sync(0xffffffffu, sec, off);
      const int ose = __shfl_xor_sync(0xffffffffu, sec_e, off);
      if (ob > best || (ob == best && oe < best_e)) {
        // theirs first; second = better of ours-first and theirs-second
        const bool mine = best > os || (best == os && best_e < ose);
        sec = mine ? best : os;
        sec_e = mine ? best_e : ose;
        best = ob;
        best_e = oe;
      } else {
        const bool mine = sec > ob || (sec == ob && sec_e < oe);
        sec = mine ? sec : ob;
        sec_e = mine ? sec_e : oe;
      }
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
      if (idx2 != nullptr) {
        idx2[t] = sec_e;
        gate2[t] = exp2f((sec - best) * kLog2e) * inv;
      }
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
                                                     o.gate, o.probs, o.psum, o.idx2, o.gate2);
  else
    router_simt_kernel<false><<<blocks, 256, sm, st>>>(T, d, N, x, w_r, b_r, logits, o.idx,
                                                      o.gate, o.probs, o.psum, o.idx2,
                                                      o.gate2);
  return cudaGetLastError();
}

// ======================================================== tensor cores

// W_r [N, d] fp32 -> bf16 terms [rows, d].  Row of (term p, expert e):
// stacked, p * N_pad + e (each term's experts together); interleaved,
// (e / 32 * terms + p) * 32 + e % 32 (the terms of 32 experts side by side,
// so one accumulator chunk of 32 x terms columns holds all of them).
// Eight consecutive elements of one row per thread: two 16-byte loads of
// W_r, one 16-byte store per term.
__global__ void wsplit_kernel(int N, int N_pad, int d, int terms, bool interleave,
                              const float* __restrict__ w_r, __nv_bfloat16* __restrict__ out) {
  // the router that follows may start its prologue and its x loads now; it
  // waits for this kernel before it reads the split
  pdl_launch_dependents();
  const int d8 = d / 8;
  const int64_t n8 = static_cast<int64_t>(N_pad) * d8;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int e = static_cast<int>(i / d8);
    const int64_t k0 = (i - static_cast<int64_t>(e) * d8) * 8;
    float w[8];
    if (e < N) {
      const float4* src = reinterpret_cast<const float4*>(w_r + static_cast<int64_t>(e) * d + k0);
      const float4 a = __ldg(src), b = __ldg(src + 1);
      w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w; w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) w[j] = 0.f;
    }
    uint32_t hi[4], mid[4], lo[4];
#pragma unroll
    for (int j = 0; j < 8; j += 2) {
      const __nv_bfloat16 h0 = __float2bfloat16_rn(w[j]), h1 = __float2bfloat16_rn(w[j + 1]);
      const float r0 = w[j] - __bfloat162float(h0), r1 = w[j + 1] - __bfloat162float(h1);   // exact
      const __nv_bfloat16 m0 = __float2bfloat16_rn(r0), m1 = __float2bfloat16_rn(r1);
      const float s0 = r0 - __bfloat162float(m0), s1 = r1 - __bfloat162float(m1);           // exact
      hi[j / 2] = pack_bf16x2(__bfloat162float(h0), __bfloat162float(h1));
      mid[j / 2] = pack_bf16x2(__bfloat162float(m0), __bfloat162float(m1));
      lo[j / 2] = pack_bf16x2(s0, s1);                    // exact: <= 8 bits each
    }
    auto row = [&](int p) -> int64_t {
      return interleave ? static_cast<int64_t>((e >> 5) * terms + p) * 32 + (e & 31)
                        : static_cast<int64_t>(p) * N_pad + e;
    };
    *reinterpret_cast<uint4*>(out + row(0) * d + k0) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(out + row(1) * d + k0) = make_uint4(mid[0], mid[1], mid[2], mid[3]);
    if (terms == 3)
      *reinterpret_cast<uint4*>(out + row(2) * d + k0) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  }
}

struct RouterTcParams {
  int64_t T;
  int d, N, N_pad, acc_stride, terms, ntiles, subs;
  int xstages, wstages;
  uint32_t wstage_bytes, tmem_cols;
  const float* b_r;
  RouterOut o;
  DevErr* err;
  long long spin;
};

// warp 0 TMA, warp 1 MMA, warps 2-9 epilogue (two groups of four)
constexpr int kRouterThreads = 64 + 256;
constexpr int kRouterMaxXStages = 12;
constexpr int kRouterMaxWStages = 4;

__device__ __forceinline__ void transpose_reduce32(float* v, int lane) {
  // After this, lane j holds in v[0] the sum over the warp's lanes of v[j].
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

// What the epilogue of a 128-token tile needs.
struct RouterEpi {
  int64_t T;
  int N, N_pad, ntiles;
  bool has_bias;
  const float* bias_s;     // [N_pad] in shared memory
  RouterOut o;
};

// Logits of experts 32c .. 32c + 31 of this thread's token: the sum of the
// weight terms' accumulator columns (term p at column p * NCH * 32).
template <int NCH, int TERMS>
__device__ __forceinline__ void load_logits(uint32_t taddr, int c, float* v) {
  tmem_ld32(taddr + c * 32, v);
#pragma unroll
  for (int p = 1; p < TERMS; ++p) {
    float w[32];
    tmem_ld32(taddr + p * NCH * 32 + c * 32, w);
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] += w[j];
  }
}

// Softmax of one token (this thread's TMEM lane) of a 128-token tile, in
// three streaming passes over its logits in TMEM, 32 values live at a time:
// the max; the sum of exponentials and the first index of the max; the
// scaled probabilities (stored when asked) and the warp's column sums of
// them into redq[e] (a butterfly transpose-reduce over the warp's 32
// tokens).  All TMEM reads of the tile are done when this returns.
template <int NCH, int TERMS>
__device__ __forceinline__ void router_softmax(const RouterEpi& ep, uint32_t taddr, int64_t t,
                                               float* redq, int lane, int& best_out,
                                               float& inv_out) {
  const bool valid = t < ep.T;
  const int N = ep.N;
  float v[32];
  float m = -INFINITY;
#pragma unroll 1
  for (int c = 0; c < NCH; ++c) {
    load_logits<NCH, TERMS>(taddr, c, v);
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float hv = ep.has_bias ? v[j] + ep.bias_s[c * 32 + j] : v[j];
      if (c * 32 + j < N) m = fmaxf(m, hv);
    }
  }
  const float mL = m * kLog2e;
  float s4[4] = {0.f, 0.f, 0.f, 0.f};
  int best = 0x7fffffff;
#pragma unroll 1
  for (int c = 0; c < NCH; ++c) {
    load_logits<NCH, TERMS>(taddr, c, v);
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int e = c * 32 + j;
      const float hv = ep.has_bias ? v[j] + ep.bias_s[e] : v[j];
      if (e < N) {
        s4[j & 3] += exp2_fast(fmaf(hv, kLog2e, -mL));
        if (hv == m && e < best) best = e;
      }
    }
  }
  const float inv = 1.f / ((s4[0] + s4[1]) + (s4[2] + s4[3]));
  const float scale = valid ? inv : 0.f;
#pragma unroll 1
  for (int c = 0; c < NCH; ++c) {
    load_logits<NCH, TERMS>(taddr, c, v);
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int e = c * 32 + j;
      const float hv = ep.has_bias ? v[j] + ep.bias_s[e] : v[j];
      v[j] = e < N ? exp2_fast(fmaf(hv, kLog2e, -mL)) * scale : 0.f;
    }
    if (valid && ep.o.probs != nullptr) {
      float* dst = ep.o.probs + t * N + c * 32;
      if ((N % 4) == 0 && c * 32 + 32 <= N) {
#pragma unroll
        for (int j = 0; j < 32; j += 4)
          *reinterpret_cast<float4*>(dst + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (c * 32 + j < N) dst[j] = v[j];
      }
    }
    transpose_reduce32(v, lane);
    redq[c * 32 + lane] = v[0];
  }
  best_out = best;
  inv_out = inv;
}

// The rest of a tile's epilogue, by its four warps (128 threads, named
// barrier `bar`; warp quarter q holds tokens 32q .. 32q + 31): idx and gate,
// each token's rank among the tile's tokens with the same expert (token
// order), the tile's histogram and its column sums of the probabilities.
__device__ __forceinline__ void router_finish(const RouterEpi& ep, int tile, int64_t t, int best,
                                              float inv, int q, int lane, int et, int bar,
                                              const float* redg, int* cntg) {
  const bool valid = t < ep.T;
  const int N = ep.N, N_pad = ep.N_pad;
  for (int i = et; i < 4 * N_pad; i += 128) cntg[i] = 0;
  named_bar_sync(bar, 128);
  if (valid) {
    ep.o.idx[t] = best;
    ep.o.gate[t] = inv;
  }
  const int e_key = valid ? best : -1;
  const unsigned peers = __match_any_sync(0xffffffffu, e_key);
  const int rank_w = __popc(peers & ((1u << lane) - 1u));
  if (valid && rank_w == 0) cntg[q * N_pad + best] = __popc(peers);
  named_bar_sync(bar, 128);
  if (valid && ep.o.local_rank != nullptr) {
    int r = rank_w;
    for (int qq = 0; qq < q; ++qq) r += cntg[qq * N_pad + best];
    ep.o.local_rank[t] = r;
  }
  for (int e = et; e < N; e += 128) {
    if (ep.o.psum != nullptr)
      ep.o.psum[static_cast<int64_t>(tile) * N + e] =
          ((redg[e] + redg[N_pad + e]) + redg[2 * N_pad + e]) + redg[3 * N_pad + e];
    if (ep.o.hist != nullptr)
      ep.o.hist[static_cast<int64_t>(e) * ep.ntiles + tile] =
          cntg[e] + cntg[N_pad + e] + cntg[2 * N_pad + e] + cntg[3 * N_pad + e];
  }
  named_bar_sync(bar, 128);
}

// Each CTA owns `subs` consecutive 128-token tiles, all accumulated at once
// (subs x N_pad fp32 TMEM columns).  The K loop is outermost: every k-block
// of the split router weight is loaded into shared memory once per CTA and
// used for all its tiles, so the weight is read from L2 once per CTA rather
// than once per tile; x streams through a deeper ring of its own.
template <int NCH, int TERMS>
__global__ void __launch_bounds__(kRouterThreads, 1) router_tc_kernel(
    const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
    RouterTcParams prm) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const int XS = prm.xstages, WS = prm.wstages, SUBS = prm.subs;
  const int N = prm.N, N_pad = prm.N_pad, NS = prm.acc_stride;
  constexpr uint32_t kXBytes = 128 * 128;                // one 128-token x block
  uint8_t* xring = smem;
  uint8_t* wring = smem + static_cast<size_t>(XS) * kXBytes;
  uint8_t* tail = wring + static_cast<size_t>(WS) * prm.wstage_bytes;
  uint64_t* xfull = reinterpret_cast<uint64_t*>(tail);
  uint64_t* xempty = xfull + kRouterMaxXStages;
  uint64_t* wfull = xempty + kRouterMaxXStages;
  uint64_t* wempty = wfull + kRouterMaxWStages;
  uint64_t* tfull = wempty + kRouterMaxWStages;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tfull + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* epi_abort = abort_flag + 1;              // [2] one per epilogue group
  float* bias_s = reinterpret_cast<float*>(tail + 512);  // [N_pad]
  float* red = bias_s + N_pad;                           // [2][4][N_pad]
  int* cnt = reinterpret_cast<int*>(red + 2 * 4 * N_pad);   // [2][4][N_pad]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kblocks = prm.d / 64;
  const long long lim = prm.spin;
  const int tile0 = blockIdx.x * SUBS;
  const int ntile_here = min(SUBS, prm.ntiles - tile0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < XS; ++s) {
      mbar_init(&xfull[s], 1);
      mbar_init(&xempty[s], 1);
    }
    for (int s = 0; s < WS; ++s) {
      mbar_init(&wfull[s], 1);
      mbar_init(&wempty[s], 1);
    }
    mbar_init(tfull, 1);
    *abort_flag = 0;
    epi_abort[0] = 0;
    epi_abort[1] = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  for (int i = threadIdx.x; i < N_pad; i += blockDim.x)
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
      int xs = 0, ws = 0;
      uint32_t xph = 0, wph = 0;
      uint32_t xmask = 0, xphs = 0, wmask = 0, wphs = 0;
      bool ok = true;
      for (int kb = 0; kb < kblocks && ok; ++kb) {
        if (!mbar_wait(&wempty[ws], wph ^ 1u, lim)) { ok = false; break; }
        mbar_arrive_expect_tx(&wfull[ws], prm.wstage_bytes);
        uint8_t* wb = wring + static_cast<size_t>(ws) * prm.wstage_bytes;
        for (int p = 0; p < prm.terms; ++p)
          tma_load_2d(wb + static_cast<size_t>(p) * N_pad * 128, &tmap_w, &wfull[ws], kb * 64,
                      p * N_pad);
        wmask |= 1u << ws;
        wphs = (wphs & ~(1u << ws)) | (wph << ws);
        if (++ws == WS) { ws = 0; wph ^= 1u; }
        for (int s = 0; s < ntile_here; ++s) {
          if (!mbar_wait(&xempty[xs], xph ^ 1u, lim)) { ok = false; break; }
          mbar_arrive_expect_tx(&xfull[xs], kXBytes);
          tma_load_2d(xring + static_cast<size_t>(xs) * kXBytes, &tmap_x, &xfull[xs], kb * 64,
                      (tile0 + s) * 128);
          xmask |= 1u << xs;
          xphs = (xphs & ~(1u << xs)) | (xph << xs);
          if (++xs == XS) { xs = 0; xph ^= 1u; }
        }
      }
      if (!ok) {
        report_error(prm.err, SWITCH_ERR_TIMEOUT, kWhereRouterProducer, blockIdx.x);
        *abort_flag = 1;
      }
      // Never leave with copies in flight into this CTA's shared memory.
      for (int s = 0; s < XS; ++s)
        if (((xmask >> s) & 1u) && !mbar_wait(&xfull[s], (xphs >> s) & 1u, kDefaultSpinCycles))
          report_error(prm.err, SWITCH_ERR_TIMEOUT, kWhereDrain, s);
      for (int s = 0; s < WS; ++s)
        if (((wmask >> s) & 1u) && !mbar_wait(&wfull[s], (wphs >> s) & 1u, kDefaultSpinCycles))
          report_error(prm.err, SWITCH_ERR_TIMEOUT, kWhereDrain, s);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      // Terms are stacked along the MMA's N dimension (each term has its own
      // N_PAD accumulator columns), GSIZE terms per instruction.
      constexpr int N_PAD = NCH * 32;
      constexpr int GSIZE = (256 / N_PAD) < TERMS ? (256 / N_PAD) : TERMS;
      constexpr int NGROUPS = (TERMS + GSIZE - 1) / GSIZE;
      constexpr int LAST = TERMS - (NGROUPS - 1) * GSIZE;
      constexpr uint32_t idesc_full = idesc_bf16_f32(128, GSIZE * N_PAD);
      constexpr uint32_t idesc_last = idesc_bf16_f32(128, LAST * N_PAD);
      int xs = 0, ws = 0;
      uint32_t xph = 0, wph = 0;
      bool ok = true, any = false;
      // Descriptors are built once per ring slot and advanced by constants
      // (the start-address field counts 16-byte units): the MMA issue loop
      // must stay well under the 64 tensor-core cycles of one MMA.
      const uint64_t xdesc0 = sw128_kmajor_desc(smem_u32(xring));
      const uint64_t wdesc0 = sw128_kmajor_desc(smem_u32(wring));
      const uint64_t term_step = static_cast<uint64_t>(N_pad * 128 / 16);
      for (int kb = 0; kb < kblocks && ok && !*abort_flag; ++kb) {
        if (!mbar_wait(&wfull[ws], wph, lim)) { ok = false; break; }
        tc_fence_after();
        const uint64_t wd = wdesc0 + static_cast<uint64_t>(ws) * (prm.wstage_bytes / 16);
        for (int s = 0; s < ntile_here; ++s) {
          if (!mbar_wait(&xfull[xs], xph, lim)) { ok = false; break; }
          tc_fence_after();
          const uint64_t xd = xdesc0 + static_cast<uint64_t>(xs) * (kXBytes / 16);
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(s * NS);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
#pragma unroll
            for (int g = 0; g < NGROUPS; ++g)
              umma_bf16(d_tmem + static_cast<uint32_t>(g * GSIZE * N_PAD), xd + 2 * k,
                        wd + g * GSIZE * term_step + 2 * k,
                        g == NGROUPS - 1 ? idesc_last : idesc_full, (kb | k) != 0 ? 1u : 0u);
          }
          any = true;
          umma_commit(&xempty[xs]);
          if (++xs == XS) { xs = 0; xph ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&wempty[ws]);
        if (++ws == WS) { ws = 0; wph ^= 1u; }
      }
      if (!ok) {
        report_error(prm.err, SWITCH_ERR_TIMEOUT, kWhereRouterMma, blockIdx.x);
        *abort_flag = 1;
      }
      // Accumulators complete (or, after an error, every issued MMA done):
      // the epilogue may read TMEM, and TMEM may be released.
      if (any || ok) umma_commit(tfull);
      else mbar_arrive(tfull);
      // After an error nobody else may wait for the MMAs: do it here, so
      // TMEM is never released under an MMA still in flight.
      if ((!ok || *abort_flag) && !mbar_wait(tfull, 0, kDefaultSpinCycles))
        report_error(prm.err, SWITCH_ERR_TIMEOUT, kWhereDrain, -1);
    }
  } else {
    // ------------------------------------------------------- epilogue
    // group g (warps 2-5: g = 0, warps 6-9: g = 1) takes tiles g, g + 2, ...
    // of the CTA; each warp owns the 32 TMEM lanes (tokens) of its quarter.
    const int g = (warp - 2) >> 2;
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int et = (threadIdx.x - 64) & 127;
    float* redg = red + g * 4 * N_pad;
    int* cntg = cnt + g * 4 * N_pad;
    volatile int* my_abort = epi_abort + g;
    const bool ok = mbar_wait_sleepy(tfull, 0, lim);
    if (!ok || *abort_flag) *my_abort = 1;
    named_bar_sync(1 + g, 128);
    if (*my_abort) {
      if (et == 0) report_error(prm.err, SWITCH_ERR_TIMEOUT, kWhereRouterEpilogue, blockIdx.x);
    } else {
      tc_fence_after();
      const RouterEpi ep{prm.T, N, N_pad, prm.ntiles, prm.b_r != nullptr, bias_s, prm.o};
      for (int s = g; s < ntile_here; s += 2) {
        const int tile = tile0 + s;
        const int64_t t = static_cast<int64_t>(tile) * 128 + row;
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                               static_cast<uint32_t>(s * NS);
        int best;
        float inv;
        router_softmax<NCH, TERMS>(ep, taddr, t, redg + q * N_pad, lane, best, inv);
        router_finish(ep, tile, t, best, inv, q, lane, et, 1 + g, redg, cntg);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, prm.tmem_cols);
}

// ---------------------------------------------------------- CTA pairs
//
// Persistent router on CTA pairs with double-buffered accumulators, for
// terms x N_pad <= 256 (one MMA covers every expert and every weight term).
// A pair tile is 256 tokens: CTA r holds tokens 128 r .. 128 r + 127 (the A
// operand) and half of the stacked weight split (rows r * Nt/2 .. of the
// B operand, Nt = terms x N_pad; with two terms, one term per CTA).  The
// leader issues tcgen05.mma.cta_group::2 (M = 256, N = Nt, K = 16); each
// CTA's TMEM receives its 128 tokens x all Nt columns.  Every SM streams 16 KB
// of x and Nt/2 x 128 B of weights per 64-deep K step.  x comes from DRAM
// and the weights from L2, so they have rings of their own: a deep one for x
// (the bytes in flight that DRAM's latency needs) and a shallow one for the
// weights, each filled by its own producer thread.  Two TMEM accumulators
// alternate between tiles; all eight epilogue warps drain every tile, so the
// softmax of one tile overlaps the main loop of the next.
struct RouterPairParams {
  int64_t T;
  int d, N, N_pad, ntiles, npairs, xstages, wstages;
  uint32_t x_bytes, w_bytes;       // per stage and CTA
  int w_half_rows;
  const float* b_r;
  RouterOut o;
  DevErr* err;
  long long spin;
};

constexpr int kRouterPairMaxXStages = 12;
constexpr int kRouterPairMaxWStages = 10;
// warp 0 x producer, warp 1 MMA, warp 2 weight producer, warps 3-10 epilogue
constexpr int kRouterPairThreads = 96 + 256;

template <int NCH, int TERMS>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kRouterPairThreads, 1)
    router_pair_kernel(const __grid_constant__ CUtensorMap tmap_x,
                       const __grid_constant__ CUtensorMap tmap_w, RouterPairParams prm) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const int XST = prm.xstages, WST = prm.wstages;
  const int N = prm.N, N_pad = prm.N_pad;
  constexpr int NT = NCH * 32 * TERMS;                   // accumulator columns per tile
  uint8_t* wring = smem + static_cast<size_t>(XST) * prm.x_bytes;
  uint8_t* tail = wring + static_cast<size_t>(WST) * prm.w_bytes;
  uint64_t* xfull = reinterpret_cast<uint64_t*>(tail);   // leader: x bytes of both CTAs
  uint64_t* xempty = xfull + kRouterPairMaxXStages;      // local: x stage consumed
  uint64_t* wfull = xempty + kRouterPairMaxXStages;      // leader: weight bytes of both CTAs
  uint64_t* wempty = wfull + kRouterPairMaxWStages;      // local: weight stage consumed
  uint64_t* tfull = wempty + kRouterPairMaxWStages;      // local: accumulator g ready
  uint64_t* tempty = tfull + 2;                          // leader: accumulator g drained
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* epi_fail = abort_flag + 1;   // [2] by tile parity: an epilogue wait gave up
  float* bias_s = reinterpret_cast<float*>(tail + 512);  // [N_pad]
  float* red = bias_s + N_pad;                           // [2 parity][4 quarter][N_pad]
  int* cnt = reinterpret_cast<int*>(red + 2 * 4 * N_pad);   // [2 parity][4 quarter][N_pad]
  float* xm = reinterpret_cast<float*>(cnt + 2 * 4 * N_pad);  // [2 parity][2 half][128]
  float* xs = xm + 2 * 2 * 128;
  int* xb = reinterpret_cast<int*>(xs + 2 * 2 * 128);
  float* xm2 = reinterpret_cast<float*>(xb + 2 * 2 * 128);      // top-2: the half's second
  int* xb2 = reinterpret_cast<int*>(xm2 + 2 * 2 * 128);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cid = static_cast<int>(cluster_id_x());
  const int ncl = static_cast<int>(cluster_count_x());
  const int kblocks = prm.d / 64;
  const long long lim = prm.spin;

  if (threadIdx.x == 0) {
    for (int s = 0; s < XST; ++s) {
      mbar_init(&xfull[s], 1);
      mbar_init(&xempty[s], 1);
    }
    for (int s = 0; s < WST; ++s) {
      mbar_init(&wfull[s], 1);
      mbar_init(&wempty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 16);            // 8 epilogue warps x 2 CTAs
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    epi_fail[0] = 0;
    epi_fail[1] = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  for (int i = threadIdx.x; i < N_pad; i += blockDim.x)
    bias_s[i] = (prm.b_r != nullptr && i < N) ? prm.b_r[i] : 0.f;
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, 2 * 256);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();                          // the peer's barriers exist before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const uint32_t xfull_lead = map_to_rank(smem_u32(xfull), 0);
  const uint32_t wfull_lead = map_to_rank(smem_u32(wfull), 0);
  const uint32_t tempty_lead = map_to_rank(smem_u32(tempty), 0);

  if (warp == 0 || warp == 2) {
    // ------------------------------------------- TMA producers (x; weights)
    if (lane == 0) {
      const bool is_x = warp == 0;
      const int nst = is_x ? XST : WST;
      uint64_t* fullb = is_x ? xfull : wfull;
      uint64_t* emptyb = is_x ? xempty : wempty;
      const uint32_t full_lead = is_x ? xfull_lead : wfull_lead;
      const uint32_t bytes = is_x ? prm.x_bytes : prm.w_bytes;
      uint8_t* ring = is_x ? smem : wring;
      tma_prefetch_desc(is_x ? &tmap_x : &tmap_w);
      // the weight split is the previous kernel's output (launched as a
      // programmatic dependent of it, this kernel may be running already)
      if (!is_x) pdl_wait_prerequisites();
      int stage = 0;
      uint32_t phase = 0, issued_mask = 0, issued_phase = 0;
      bool ok = true;
      for (int pt = cid; pt < prm.npairs && ok && !*abort_flag; pt += ncl) {
        const int row = is_x ? pt * 256 + static_cast<int>(rank) * 128
                             : static_cast<int>(rank) * prm.w_half_rows;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&emptyb[stage], phase ^ 1u, lim)) { ok = false; break; }
          if (leader) mbar_arrive_expect_tx(&fullb[stage], 2 * bytes);
          tma_load_2d_pair(ring + static_cast<size_t>(stage) * bytes, is_x ? &tmap_x : &tmap_w,
                           full_lead + 8u * stage, kb * 64, row);
          issued_mask |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == nst) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        report_error(prm.err, SWITCH_ERR_TIMEOUT, kWhereRouterProducer, blockIdx.x);
        *abort_flag = 1;
      }
      // Both CTAs' bytes land on the leader's barriers: the leader waits for
      // every issued stage before the final cluster barrier.
      if (leader)
        for (int s = 0; s < nst; ++s)
          if (((issued_mask >> s) & 1u) &&
              !mbar_wait_cluster(&fullb[s], (issued_phase >> s) & 1u, kDefaultSpinCycles))
            report_error(prm.err, SWITCH_ERR_TIMEOUT, kWhereDrain, s);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (leader && lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(256, NT);
      int xs = 0, ws = 0;
      uint32_t xph = 0, wph = 0;
      bool ok = true, any = false;
      int li = 0;                                        // local tile count
      for (int pt = cid; pt < prm.npairs && ok && !*abort_flag; pt += ncl, ++li) {
        const int acc = li & 1;
        const uint32_t use = static_cast<uint32_t>(li >> 1);   // earlier uses of `acc`
        if (!mbar_wait_cluster(&tempty[acc], (use & 1u) ^ 1u, lim)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * 256);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait_cluster(&xfull[xs], xph, lim) ||
              !mbar_wait_cluster(&wfull[ws], wph, lim)) { ok = false; break; }
          tc_fence_after();
          const uint64_t xd = sw128_kmajor_desc(smem_u32(smem + static_cast<size_t>(xs) * prm.x_bytes));
          const uint64_t wd = sw128_kmajor_desc(smem_u32(wring + static_cast<size_t>(ws) * prm.w_bytes));
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16_pair(d_tmem, xd + 2 * k, wd + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
          any = true;
          umma_commit_pair(&xempty[xs], 0x3);
          umma_commit_pair(&wempty[ws], 0x3);
          if (++xs == XST) { xs = 0; xph ^= 1u; }
          if (++ws == WST) { ws = 0; wph ^= 1u; }
        }
        if (!ok) break;
        umma_commit_pair(&tfull[acc], 0x3);
      }
      if (!ok) {
        report_error(prm.err, SWITCH_ERR_TIMEOUT, kWhereRouterMma, blockIdx.x);
        *abort_flag = 1;
      }
      if (any && *abort_flag) {
        umma_commit_pair(drain, 0x1);
        if (!mbar_wait(drain, 0, kDefaultSpinCycles))
          report_error(prm.err, SWITCH_ERR_TIMEOUT, kWhereDrain, -1);
      }
    }
  } else {
    // ------------------------------------------------------- epilogue
    // All eight warps drain every tile: warp quarter q = warp % 4 owns TMEM
    // lanes (tokens) 32q .. 32q + 31, half h = (warp - 2) / 4 owns expert
    // chunks h * NH .. of them.  One TMEM pass per thread (its token's logits
    // of its half, all weight terms), after which the accumulator is handed
    // back; the halves then exchange (max, sum of exponentials, first index
    // of the max) through shared memory.  Per-tile shared arrays alternate
    // with the tile's parity.
    constexpr int NH = (NCH + 1) / 2;                  // chunks per half
    const int q = warp & 3;
    const int h = (warp - 3) >> 2;
    const int row = q * 32 + lane;
    const int et = threadIdx.x - 96;                   // 0 .. 255
    const int N_h = N - h * NH * 32;                   // experts of this half (may be <= 0)
    int li = 0;
    for (int pt = cid; pt < prm.npairs; pt += ncl, ++li) {
      const int acc = li & 1;
      // One outcome for all eight warps (they meet at named barriers below):
      // a warp whose wait gave up raises this tile's flag before the
      // barrier, every warp reads it after.  No warp gets a whole tile ahead
      // of another (each tile passes this barrier), so alternating two
      // flags keeps a later tile's failure out of this tile's decision.
      const bool ok = __all_sync(0xffffffffu,
                                 mbar_wait_sleepy(&tfull[acc], static_cast<uint32_t>(li >> 1) & 1u, lim));
      if (!ok && lane == 0) epi_fail[li & 1] = 1;
      named_bar_sync(1, 256);
      if (epi_fail[li & 1]) {
        if (et == 0) {
          report_error(prm.err, SWITCH_ERR_TIMEOUT, kWhereRouterEpilogue, blockIdx.x);
          *abort_flag = 1;
        }
        break;
      }
      tc_fence_after();
      const int tile = pt * 2 + static_cast<int>(rank);   // this CTA's 128-token tile
      const bool here = tile < prm.ntiles;                // uniform for the CTA
      const int64_t t = static_cast<int64_t>(tile) * 128 + row;
      const bool valid = t < prm.T;
      // this half's logits (sum of the weight terms, + bias), one chunk of
      // TMEM loads in flight at a time
      float v[NH * 32];
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc * 256);
      if (here) {
        // every TMEM load of this thread's logits in flight at once, one wait
        uint32_t r[NH][TERMS][32];
#pragma unroll
        for (int cc = 0; cc < NH; ++cc) {
          const int c = h * NH + cc;
#pragma unroll
          for (int p = 0; p < TERMS; ++p)
            if (c < NCH)                                  // warp-uniform
              tmem_ld32_issue(taddr + static_cast<uint32_t>((c * TERMS + p) * 32), r[cc][p]);
        }
        // (the first wait covers every load; each call also orders its array's
        // register uses after the wait)
#pragma unroll
        for (int cc = 0; cc < NH; ++cc)
#pragma unroll
          for (int p = 0; p < TERMS; ++p)
            if (h * NH + cc < NCH) tmem_ld_wait(r[cc][p]);
#pragma unroll
        for (int cc = 0; cc < NH; ++cc) {
          const int c = h * NH + cc;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            float a = __uint_as_float(r[cc][0][j]);
#pragma unroll
            for (int p = 1; p < TERMS; ++p) a += __uint_as_float(r[cc][p][j]);
            v[cc * 32 + j] = a;
          }
          if (prm.b_r != nullptr)
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (c * 32 + j < N) v[cc * 32 + j] += bias_s[c * 32 + j];
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {                                    // TMEM of this tile no longer read
        if (leader) mbar_arrive_relaxed(&tempty[acc]);
        else mbar_arrive_remote_relaxed(tempty_lead + 8u * acc);
      }
      if (!here) continue;
      const int par = li & 1;
      float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int i = 0; i < NH * 32; ++i)
        if (i < N_h) mq[i & 3] = fmaxf(mq[i & 3], v[i]);
      const float m_h = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
      int bq[4] = {0x7fffffff, 0x7fffffff, 0x7fffffff, 0x7fffffff};
#pragma unroll
      for (int i = 0; i < NH * 32; ++i)
        if (i < N_h && v[i] == m_h) bq[i & 3] = min(bq[i & 3], i);
      const int b_h = min(min(bq[0], bq[1]), min(bq[2], bq[3]));
      // top-2: the half's largest logit other than b_h, first index of it
      float m2_h = -INFINITY;
      int b2_h = 0x7fffffff;
      if (prm.o.idx2 != nullptr) {
        float mq2[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int i = 0; i < NH * 32; ++i)
          if (i < N_h && i != b_h) mq2[i & 3] = fmaxf(mq2[i & 3], v[i]);
        m2_h = fmaxf(fmaxf(mq2[0], mq2[1]), fmaxf(mq2[2], mq2[3]));
        int bq2[4] = {0x7fffffff, 0x7fffffff, 0x7fffffff, 0x7fffffff};
#pragma unroll
        for (int i = 0; i < NH * 32; ++i)
          if (i < N_h && i != b_h && v[i] == m2_h) bq2[i & 3] = min(bq2[i & 3], i);
        b2_h = min(min(bq2[0], bq2[1]), min(bq2[2], bq2[3]));
      }
      const float mL_h = m_h * kLog2e;
      float sq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < NH * 32; ++i) {
        v[i] = i < N_h ? exp2_fast(fmaf(v[i], kLog2e, -mL_h)) : 0.f;
        sq[i & 3] += v[i];
      }
      float* xm_p = xm + par * 256;
      float* xs_p = xs + par * 256;
      int* xb_p = xb + par * 256;
      xm_p[h * 128 + row] = m_h;
      xs_p[h * 128 + row] = (sq[0] + sq[1]) + (sq[2] + sq[3]);
      xb_p[h * 128 + row] = b_h == 0x7fffffff ? b_h : h * NH * 32 + b_h;
      if (prm.o.idx2 != nullptr) {
        xm2[par * 256 + h * 128 + row] = m2_h;
        xb2[par * 256 + h * 128 + row] = b2_h == 0x7fffffff ? b2_h : h * NH * 32 + b2_h;
      }
      int* cnt_p = cnt + par * 4 * N_pad;
      for (int i = et; i < 4 * N_pad; i += 256) cnt_p[i] = 0;
      named_bar_sync(1, 256);
      // the token's max, sum and expert, the same in both halves
      const float m0 = xm_p[row], m1 = xm_p[128 + row];
      const float m = fmaxf(m0, m1);
      const float s = xs_p[row] * exp2_fast((m0 - m) * kLog2e) +
                      xs_p[128 + row] * exp2_fast((m1 - m) * kLog2e);
      const int best = m0 >= m1 ? xb_p[row] : xb_p[128 + row];
      const float inv = 1.f / s;
      // top-2: the better of the other half's first and this half's second
      // (half 0 holds the lower indices, so it wins ties)
      int second = 0;
      float gate_2 = 0.f;
      if (prm.o.idx2 != nullptr) {
        float v2;
        if (m0 >= m1) {
          const float a2 = xm2[par * 256 + row];
          v2 = a2 >= m1 ? a2 : m1;
          second = a2 >= m1 ? xb2[par * 256 + row] : xb_p[128 + row];
        } else {
          const float b2 = xm2[par * 256 + 128 + row];
          v2 = m0 >= b2 ? m0 : b2;
          second = m0 >= b2 ? xb_p[row] : xb2[par * 256 + 128 + row];
        }
        gate_2 = exp2_fast((v2 - m) * kLog2e) * inv;
      }
      const float scale = valid ? exp2_fast((m_h - m) * kLog2e) * inv : 0.f;
      float* red_p = red + par * 4 * N_pad;
#pragma unroll
      for (int cc = 0; cc < NH; ++cc) {
        const int c = h * NH + cc;
        if (c >= NCH) break;                              // warp-uniform
        float pv[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) pv[j] = v[cc * 32 + j] * scale;
        if (valid && prm.o.probs != nullptr) {
          float* dst = prm.o.probs + t * N + c * 32;
          if ((N % 4) == 0 && c * 32 + 32 <= N) {
#pragma unroll
            for (int j = 0; j < 32; j += 4)
              *reinterpret_cast<float4*>(dst + j) =
                  make_float4(pv[j], pv[j + 1], pv[j + 2], pv[j + 3]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (c * 32 + j < N) dst[j] = pv[j];
          }
        }
        transpose_reduce32(pv, lane);
        red_p[q * N_pad + c * 32 + lane] = pv[0];
      }
      // dispatch ranks within the tile (token order), by half 0
      int rank_w = 0;
      if (h == 0) {
        const int e_key = valid ? best : -1;
        const unsigned peers = __match_any_sync(0xffffffffu, e_key);
        rank_w = __popc(peers & ((1u << lane) - 1u));
        if (valid && rank_w == 0) cnt_p[q * N_pad + best] = __popc(peers);
      }
      named_bar_sync(1, 256);
      if (h == 0 && valid) {
        prm.o.idx[t] = best;
        prm.o.gate[t] = inv;
        if (prm.o.idx2 != nullptr) {
          prm.o.idx2[t] = second;
          prm.o.gate2[t] = gate_2;
        }
        if (prm.o.local_rank != nullptr) {
          int rr = rank_w;
          for (int qq = 0; qq < q; ++qq) rr += cnt_p[qq * N_pad + best];
          prm.o.local_rank[t] = rr;
        }
      }
      for (int e = et; e < N; e += 256) {
        if (prm.o.psum != nullptr)
          prm.o.psum[static_cast<int64_t>(tile) * N + e] =
              ((red_p[e] + red_p[N_pad + e]) + red_p[2 * N_pad + e]) + red_p[3 * N_pad + e];
        if (prm.o.hist != nullptr)
          prm.o.hist[static_cast<int64_t>(e) * prm.ntiles + tile] =
              cnt_p[e] + cnt_p[N_pad + e] + cnt_p[2 * N_pad + e] + cnt_p[3 * N_pad + e];
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();                          // no CTA leaves while its peer may still signal it
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, 2 * 256);
}

// ------------------------------------------------------------------ host

typedef CUresult (*PFN_encodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                    const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                    const cuuint32_t*, CUtensorMapInterleave,
                                    CUtensorMapSwizzle, CUtensorMapL2promotion,
                                    CUtensorMapFloatOOBfill);

PFN_encodeTiled get_encode_fn();   // defined in expert_ffn.cu


static int router_n_pad(int N) { return (N + 31) / 32 * 32; }

size_t router_wsplit_bytes(int N, int d) {
  return sizeof(__nv_bfloat16) * 3 * static_cast<size_t>(router_n_pad(N)) * d;
}

bool router_pair_supported(int N, int terms) { return terms * router_n_pad(N) <= 256; }

// Every weight term keeps its own accumulator columns: terms x N_pad <= 512.
bool router_tc_supported(int N, int d, int terms) {
  const int n_pad = router_n_pad(N);
  return (terms == 2 || terms == 3) && terms * n_pad <= 512 && d % 64 == 0 && d > 0;
}

template <int NCH, int TERMS>
static cudaError_t run_router_tc_t(const CUtensorMap& tx, const CUtensorMap& tw,
                                   const RouterTcParams& p, size_t smem, int grid,
                                   cudaStream_t st) {
  static size_t smem_set[64] = {};
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(&router_tc_kernel<NCH, TERMS>), smem, smem_set);
  if (e != cudaSuccess) return e;
  router_tc_kernel<NCH, TERMS><<<grid, kRouterThreads, smem, st>>>(tx, tw, p);
  return cudaGetLastError();
}

template <int NCH>
static cudaError_t run_router_tc(const CUtensorMap& tx, const CUtensorMap& tw,
                                 const RouterTcParams& p, size_t smem, int grid,
                                 cudaStream_t st) {
  return p.terms == 2 ? run_router_tc_t<NCH, 2>(tx, tw, p, smem, grid, st)
                      : run_router_tc_t<NCH, 3>(tx, tw, p, smem, grid, st);
}

template <int NCH, int TERMS>
static cudaError_t run_router_pair_t(const CUtensorMap& tx, const CUtensorMap& tw,
                                     const RouterPairParams& p, size_t smem, int grid,
                                     cudaStream_t st) {
  static size_t smem_set[64] = {};
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(&router_pair_kernel<NCH, TERMS>),
                                    smem, smem_set);
  if (e != cudaSuccess) return e;
  // launched as a programmatic dependent of the weight split: its prologue,
  // TMEM allocation and first x loads overlap that kernel
  cudaLaunchConfig_t lc{};
  lc.gridDim = dim3(grid);
  lc.blockDim = dim3(kRouterPairThreads);
  lc.dynamicSmemBytes = smem;
  lc.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  return cudaLaunchKernelEx(&lc, router_pair_kernel<NCH, TERMS>, tx, tw, p);
}

// CTA-pair router: terms x N_pad <= 256.
static cudaError_t launch_router_pair(int64_t T, int d, int N, int N_pad, int terms,
                                      const void* x, const float* b_r, const void* wsplit,
                                      RouterOut o, int ntiles, DevErr* err, long long spin,
                                      int num_sms, cudaStream_t st) {
  const int nt = terms * N_pad;
  RouterPairParams p;
  p.T = T;
  p.d = d;
  p.N = N;
  p.N_pad = N_pad;
  p.ntiles = ntiles;
  p.npairs = (ntiles + 1) / 2;
  p.w_half_rows = nt / 2;
  p.x_bytes = 128u * 128u;
  p.w_bytes = static_cast<uint32_t>(nt / 2) * 128u;
  p.b_r = b_r;
  p.o = o;
  p.err = err;
  p.spin = spin;
  const size_t tail_bytes =
      512 + sizeof(float) * N_pad * 9 + sizeof(int) * N_pad * 8 + 5 * sizeof(float) * 512;
  const size_t budget = 227 * 1024 - 1024 - tail_bytes;
  // x comes from DRAM: eight 16 KB stages (128 KB in flight per SM); the
  // weights from L2, whose latency under this load is still microseconds:
  // the rest of shared memory (the same bytes per K step as x)
  int xst = 8;
  int wst = static_cast<int>((budget - static_cast<size_t>(xst) * p.x_bytes) / p.w_bytes);
  if (wst > kRouterPairMaxWStages) wst = kRouterPairMaxWStages;
  if (wst < 2) return cudaErrorInvalidConfiguration;
  p.xstages = xst;
  p.wstages = wst;
  CUtensorMap tx, tw;
  if (!make_tmap_bf16_2d(&tx, x, static_cast<uint64_t>(d), static_cast<uint64_t>(T), 64, 128))
    return cudaErrorInvalidValue;
  if (!make_tmap_bf16_2d(&tw, wsplit, static_cast<uint64_t>(d), static_cast<uint64_t>(nt), 64,
                         static_cast<uint32_t>(nt / 2)))
    return cudaErrorInvalidValue;
  const size_t smem = 1024 + static_cast<size_t>(xst) * p.x_bytes +
                      static_cast<size_t>(wst) * p.w_bytes + tail_bytes;
  int clusters = num_sms / 2;
  if (clusters > p.npairs) clusters = p.npairs;
  if (clusters < 1) clusters = 1;
  const int grid = 2 * clusters;
  const int nch = N_pad / 32;
  if (terms == 2) {
    switch (nch) {
      case 1: return run_router_pair_t<1, 2>(tx, tw, p, smem, grid, st);
      case 2: return run_router_pair_t<2, 2>(tx, tw, p, smem, grid, st);
      case 3: return run_router_pair_t<3, 2>(tx, tw, p, smem, grid, st);
      default: return run_router_pair_t<4, 2>(tx, tw, p, smem, grid, st);
    }
  }
  switch (nch) {
    case 1: return run_router_pair_t<1, 3>(tx, tw, p, smem, grid, st);
    default: return run_router_pair_t<2, 3>(tx, tw, p, smem, grid, st);
  }
}

cudaError_t launch_router_tc(int64_t T, int d, int N, int terms, const void* x,
                             const float* w_r, const float* b_r, void* wsplit, RouterOut o,
                             int ntiles, DevErr* err, long long spin, int num_sms,
                             cudaStream_t st) {
  const int N_pad = router_n_pad(N);
  const bool pair = terms * N_pad <= 256 && num_sms >= 2;
  {
    const int64_t n8 = static_cast<int64_t>(N_pad) * (d / 8);     // d % 64 == 0
    int blocks = static_cast<int>((n8 + 127) / 128);
    if (blocks > 1024) blocks = 1024;
    wsplit_kernel<<<blocks, 128, 0, st>>>(N, N_pad, d, terms, pair, w_r,
                                          static_cast<__nv_bfloat16*>(wsplit));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (pair)
    return launch_router_pair(T, d, N, N_pad, terms, x, b_r, wsplit, o, ntiles, err, spin,
                              num_sms, st);
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
  // One tile's accumulator: the terms side by side, N_pad (a multiple of 32)
  // columns each.
  const int ns = terms * N_pad;
  p.acc_stride = ns;
  // Tiles per CTA: enough to cover the tokens in about one wave, at most
  // what TMEM holds (512 fp32 columns).
  int subs = (ntiles + num_sms - 1) / num_sms;
  if (subs > 512 / ns) subs = 512 / ns;
  if (subs < 1) subs = 1;
  p.subs = subs;
  p.wstage_bytes = static_cast<uint32_t>(terms) * N_pad * 128u;
  const size_t tail_bytes = 512 + sizeof(float) * N_pad * 9 + sizeof(int) * N_pad * 8;
  const size_t budget = 227 * 1024 - 1024 - tail_bytes;
  int wst = 2;
  int xst = static_cast<int>((budget - wst * p.wstage_bytes) / (128 * 128));
  if (xst > kRouterMaxXStages) xst = kRouterMaxXStages;
  if (xst < 2) return cudaErrorInvalidConfiguration;
  p.xstages = xst;
  p.wstages = wst;
  uint32_t cols = 32;
  while (cols < static_cast<uint32_t>(subs * ns)) cols <<= 1;
  p.tmem_cols = cols;
  p.b_r = b_r;
  p.o = o;
  p.err = err;
  p.spin = spin;
  const size_t smem = 1024 + static_cast<size_t>(xst) * 128 * 128 +
                      static_cast<size_t>(wst) * p.wstage_bytes + tail_bytes;
  const int grid = (ntiles + subs - 1) / subs;
  switch (N_pad / 32) {
    case 1: return run_router_tc<1>(tx, tw, p, smem, grid, st);
    case 2: return run_router_tc<2>(tx, tw, p, smem, grid, st);
    case 3: return run_router_tc<3>(tx, tw, p, smem, grid, st);
    case 4: return run_router_tc<4>(tx, tw, p, smem, grid, st);
    case 5: return run_router_tc<5>(tx, tw, p, smem, grid, st);
    case 6: return run_router_tc<6>(tx, tw, p, smem, grid, st);
    case 7: return run_router_tc<7>(tx, tw, p, smem, grid, st);
    default: return run_router_tc<8>(tx, tw, p, smem, grid, st);
  }
}

}  // namespace smoe
