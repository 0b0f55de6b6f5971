// C ABI of the Switch-FFN layer (declared in include/switch_moe.h):
// argument validation, exact capacity, workspace carving and the launch
// sequence of each entry point.  No device memory is allocated here.
#include <algorithm>
#include <climits>
#include <cmath>
#include <cstring>

#include "backward.cuh"

using namespace smoe;

namespace {

constexpr size_t kAlign = 1024;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ceil(T * cf / N) with cf taken at the exact value of the double.
int64_t capacity_exact(int64_t T, int32_t N, double cf) {
  if (T < 0 || N < 1 || !(cf > 0.0) || !std::isfinite(cf)) return -1;
  if (T == 0) return 0;
  int ex = 0;
  const double f = std::frexp(cf, &ex);                          // cf = f * 2^ex
  const uint64_t mant = static_cast<uint64_t>(std::ldexp(f, 53));  // exact, < 2^53
  int sh = ex - 53;                                               // cf = mant * 2^sh
  unsigned __int128 num = static_cast<unsigned __int128>(T) * mant;
  unsigned __int128 den = static_cast<unsigned __int128>(N);
  if (sh >= 0) {
    if (sh > 10) return -1;                                       // cf >= 2^63: nonsense
    num <<= sh;
  } else {
    if (-sh > 116) return 1;                                      // 0 < T cf / N < 1
    den <<= -sh;
  }
  const unsigned __int128 q = (num + den - 1) / den;
  if (q > static_cast<unsigned __int128>(INT64_MAX)) return -1;
  return static_cast<int64_t>(q);
}

struct Layout {
  size_t err, hist, base, psum, fpsc, local_rank, idx, gate, rank, drop, counts, counts1,
      slot_token, mtile_start, wsplit, logits, xdisp, hbuf, ybuf, total;
  // backward pass only (after the forward regions): dA, partial gate
  // gradients, dh (fp32, and its bf16 planes per token and per slot), W_r
  // planes, gate gradient (per route), split-K partials of dW_r, column
  // sums of dh, dropped-token list and its counter; top-2 and fp32 only:
  // the dX GEMM's fp32 rows per slot
  size_t probs_s, da, dgp, dh, dhp, dhs, wrp, dgate, rpart, colsum, drop_list, n_drop, dxs,
      bwd_total;
};

// Bytes 16..19 of the workspace: the loss kernel's completion ticket (kept
// at zero between calls, like the error word in bytes 0..15).
constexpr size_t kTicketOffset = 16;
// Bytes 32 .. 32 + 4 kAuxChunks: the staged loss's per-run tickets (also
// left at zero).
constexpr size_t kRunTicketOffset = 32;
static_assert(kRunTicketOffset + 4 * kAuxChunks <= 256, "tickets live in the first 256 bytes");

int ntiles_of(int64_t T) { return static_cast<int>((T + kTileTok - 1) / kTileTok); }

// Routes per token: 2 with SWITCH_FLAG_TOP2, else 1.  Dispatch works on the
// routes x T (token, expert) assignments, route-major.
int routes_of(const switch_config_t& c) { return (c.flags & SWITCH_FLAG_TOP2) ? 2 : 1; }

Layout layout_for(const switch_config_t& c, int64_t C) {
  const int64_t T = c.T;
  const int64_t A = routes_of(c) * T;        // assignments
  const int64_t N = c.n_experts;
  const size_t es = c.dtype == SWITCH_BF16 ? 2 : 4;
  const int64_t nt = ntiles_of(A);
  const int64_t nparts = (T + 63) / 64;
  const int64_t slots = N * C;
  Layout L{};
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + (bytes ? bytes : 1), kAlign);
    return at;
  };
  L.err = take(256);
  L.hist = take(sizeof(int) * N * nt);
  L.base = take(sizeof(int) * N * nt);
  L.psum = take(sizeof(float) * N * nparts);
  L.fpsc = take(sizeof(double) * N * kAuxChunks);
  L.local_rank = take(sizeof(int) * A);
  L.idx = take(sizeof(int) * A);
  L.gate = take(sizeof(float) * A);
  L.rank = take(sizeof(int) * A);
  L.drop = take(A);
  L.counts = take(sizeof(int) * N);
  L.counts1 = take(sizeof(int) * N);
  L.slot_token = take(sizeof(int) * slots);
  L.mtile_start = take(sizeof(int) * (N + 1));
  L.wsplit = take(router_wsplit_bytes(c.n_experts, c.d_model));
  L.logits = take(sizeof(float) * N * T);
  L.xdisp = take(es * slots * static_cast<size_t>(c.d_model));
  L.hbuf = take(es * slots * static_cast<size_t>(c.d_ff));
  L.ybuf = take(es * slots * static_cast<size_t>(c.d_model));
  L.total = o;
  const int64_t ntn = (c.d_ff + 255) / 256;
  L.probs_s = take(sizeof(float) * N * T);      // router probabilities kept for the backward
  L.da = take(es * slots * static_cast<size_t>(c.d_ff));
  // gate-gradient partials: one per 256 columns (bf16 tiles) or 64 (fp32)
  L.dgp = take(sizeof(float) * slots * std::max<int64_t>(ntn, (c.d_ff + 63) / 64));
  const int64_t Np = (N + 63) / 64 * 64;
  L.dh = take(sizeof(float) * N * T);
  L.dhp = take(2 * 2 * static_cast<size_t>(T) * Np);
  L.dhs = take(2 * 2 * static_cast<size_t>(slots) * Np);
  L.wrp = take(2 * 2 * static_cast<size_t>(Np) * c.d_model);
  L.dgate = take(sizeof(float) * A);
  L.rpart = take(sizeof(float) * router_bwd_tc_part_floats(T, c.n_experts, c.d_model, 0));
  L.colsum = take(sizeof(float) * N * ntiles_of(T));
  L.drop_list = take(sizeof(int) * T);
  L.n_drop = take(sizeof(int));
  L.dxs = take(routes_of(c) == 2 || c.dtype != SWITCH_BF16
                   ? sizeof(float) * slots * static_cast<size_t>(c.d_model)
                   : 0);
  L.bwd_total = o;
  return L;
}

switch_status_t validate(const switch_config_t* c, int64_t* C_out) {
  if (c == nullptr) return SWITCH_ERR_INVALID_ARG;
  if (c->T < 0 || c->T > INT_MAX || c->d_model < 1 || c->d_ff < 1 || c->n_experts < 1 ||
      c->n_experts > 1024 || (c->dtype != SWITCH_F32 && c->dtype != SWITCH_BF16) ||
      c->spin_limit < 0)
    return SWITCH_ERR_INVALID_ARG;
  if ((c->flags & SWITCH_FLAG_TOP2) && (c->n_experts < 2 || c->T > INT_MAX / 2))
    return SWITCH_ERR_INVALID_ARG;
  // capacity over the routes x T assignments: each expert takes tokens from
  // every route
  const int64_t C = capacity_exact(routes_of(*c) * c->T, c->n_experts, c->capacity_factor);
  if (C < 0) return SWITCH_ERR_INVALID_ARG;
  if (c->dtype == SWITCH_BF16 && (c->d_model % 64 != 0 || c->d_ff % 64 != 0))
    return SWITCH_ERR_UNSUPPORTED;
  if (c->dtype == SWITCH_F32 && (c->d_model % 4 != 0 || c->d_ff % 4 != 0))
    return SWITCH_ERR_UNSUPPORTED;
  if (C > INT_MAX / c->n_experts) return SWITCH_ERR_UNSUPPORTED;   // slot ids are int32
  if (C_out) *C_out = C;
  return SWITCH_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Ctx {
  int64_t C;
  Layout L;
  uint8_t* ws;
  DevErr* err;
  cudaStream_t st;
  long long spin;
  int num_sms;
  template <class P>
  P* at(size_t off) const { return reinterpret_cast<P*>(ws + off); }
};

int device_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cache[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    int major = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cache[dev] = major == 10 ? v : -1;   // the kernels are built for sm_100a only
  }
  return cache[dev];
}

switch_status_t prepare(const switch_config_t* cfg, void* ws, size_t ws_bytes, void* stream,
                        Ctx* ctx) {
  int64_t C = 0;
  switch_status_t s = validate(cfg, &C);
  if (s != SWITCH_OK) return s;
  ctx->C = C;
  ctx->L = layout_for(*cfg, C);
  if (cfg->T == 0) return SWITCH_OK;
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
    return SWITCH_ERR_INVALID_ARG;
  if (ws_bytes < ctx->L.total) return SWITCH_ERR_WORKSPACE_TOO_SMALL;
  ctx->ws = static_cast<uint8_t*>(ws);
  ctx->err = reinterpret_cast<DevErr*>(ws);
  ctx->st = static_cast<cudaStream_t>(stream);
  ctx->spin = cfg->spin_limit > 0 ? cfg->spin_limit : kDefaultSpinCycles;
  ctx->num_sms = device_sms();
  if (ctx->num_sms == 0) return SWITCH_ERR_CUDA;
  if (ctx->num_sms < 0) return SWITCH_ERR_UNSUPPORTED;
  return SWITCH_OK;
}

switch_status_t cuda_status(cudaError_t e) {
  return e == cudaSuccess ? SWITCH_OK : SWITCH_ERR_CUDA;
}

#define SMOE_TRY(expr)                         \
  do {                                         \
    cudaError_t _e = (expr);                   \
    if (_e != cudaSuccess) return SWITCH_ERR_CUDA; \
  } while (0)

// GEMM1 on row-major CTA pairs (each SM streams a third fewer operand bytes
// per K step; an expert's last 128 rows take a half tile, not a padded pair
// tile): asked for, or by default when C > 128 and either every expert's
// rows fit one pair tile (C <= 256) or d_model >= 2048, where a tile's long
// K loop amortises its epilogue (measured: XXL 1364-1376 vs 1394-1422 us;
// with d_model 768 and C 512-1024 the one-CTA kernel is as fast or 1.5%
// faster).
bool gemm1_rows_pairs(const switch_config_t* c, int64_t C) {
  if (c->flags & SWITCH_FLAG_GEMM1_ROWS_PAIRS) return true;
  if (c->flags & (SWITCH_FLAG_GEMM_1SM | SWITCH_FLAG_GEMM_PAIRS | SWITCH_FLAG_GATHER_IN_GEMM))
    return false;
  return C > 128 && (C <= 256 || c->d_model >= 2048);
}

int router_terms(const switch_config_t* c) {
  return (c->flags & SWITCH_FLAG_ROUTER_3TERM) ? 3 : 2;
}

// Tensor-core router; top-2 only on the CTA-pair kernel (terms x N_pad <= 256).
bool use_tc_router(const switch_config_t* c) {
  return c->dtype == SWITCH_BF16 && !(c->flags & SWITCH_FLAG_ROUTER_SIMT) &&
         router_tc_supported(c->n_experts, c->d_model, router_terms(c)) &&
         (!(c->flags & SWITCH_FLAG_TOP2) || router_pair_supported(c->n_experts, router_terms(c)));
}

// ------------------------------------------------------ expert parallelism

// Regions of one rank's expert-parallel workspace, of the record every rank
// all-gathers, and of the receive buffer peers store into.
struct EpLayout {
  int G, r, e_loc, nt, nparts, nparts_max;
  int64_t T, C;
  bool tc_router;
  size_t err, hist, base, local_rank, idx, gate, rank, drop, wsplit, logits, psum_cat,
      counts_glob, counts_loc, mtile_start, fpsc, hbuf, total;
  size_t payload_counts, payload_total;       // record: psum parts, then counts
  size_t recv_src, recv_gate, recv_total;     // receive: rows, sources, gates
};

switch_status_t ep_layout(const switch_config_t* c, const switch_ep_t* ep, EpLayout* L) {
  if (c == nullptr || ep == nullptr) return SWITCH_ERR_INVALID_ARG;
  const int G = ep->world_size;
  if (G < 1 || G > kEpMaxRanks || ep->rank < 0 || ep->rank >= G) return SWITCH_ERR_INVALID_ARG;
  if (c->T < 0 || c->T >= (int64_t{1} << kEpRankShift) || c->T * G > INT_MAX)
    return SWITCH_ERR_UNSUPPORTED;
  switch_config_t whole = *c;                 // the global batch: G ranks' tokens
  whole.T = c->T * G;
  int64_t C = 0;
  switch_status_t s = validate(&whole, &C);
  if (s != SWITCH_OK) return s;
  if (c->dtype != SWITCH_BF16 || (c->flags & (SWITCH_FLAG_TOP2 | SWITCH_FLAG_GEMM_1SM)) ||
      c->n_experts % G != 0)
    return SWITCH_ERR_UNSUPPORTED;
  *L = EpLayout{};
  L->G = G;
  L->r = ep->rank;
  L->e_loc = c->n_experts / G;
  L->T = c->T;
  L->C = C;
  L->nt = ntiles_of(c->T);
  L->tc_router = use_tc_router(c);
  L->nparts_max = static_cast<int>((c->T + 63) / 64);
  L->nparts = L->tc_router ? L->nt : L->nparts_max;
  const int64_t N = c->n_experts, T = c->T;
  const int64_t S = static_cast<int64_t>(L->e_loc) * C;    // this rank's slots
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + (bytes ? bytes : 1), kAlign);
    return at;
  };
  L->err = take(256);
  L->hist = take(sizeof(int) * N * L->nt);
  L->base = take(sizeof(int) * N * L->nt);
  L->local_rank = take(sizeof(int) * T);
  L->idx = take(sizeof(int) * T);
  L->gate = take(sizeof(float) * T);
  L->rank = take(sizeof(int) * T);
  L->drop = take(T);
  L->wsplit = take(router_wsplit_bytes(c->n_experts, c->d_model));
  L->logits = take(L->tc_router ? 0 : sizeof(float) * N * T);
  L->psum_cat = take(sizeof(float) * N * L->nparts * G);
  L->counts_glob = take(sizeof(int) * N);
  L->counts_loc = take(sizeof(int) * L->e_loc);
  L->mtile_start = take(sizeof(int) * (L->e_loc + 1));
  L->fpsc = take(sizeof(double) * N * kAuxChunks);
  L->hbuf = take(2 * static_cast<size_t>(S) * c->d_ff);
  L->total = o;
  L->payload_counts = align_up(sizeof(float) * N * L->nparts_max, 16);
  L->payload_total = align_up(L->payload_counts + sizeof(int) * N, 16);
  L->recv_src = align_up(2 * static_cast<size_t>(S) * c->d_model, 256);
  L->recv_gate = align_up(L->recv_src + sizeof(int) * S, 256);
  L->recv_total = align_up(L->recv_gate + sizeof(float) * S, 256);
  return SWITCH_OK;
}

// Workspace checks shared by the expert-parallel calls.
switch_status_t ep_prepare_call(const switch_config_t* cfg, const switch_ep_t* ep, void* ws,
                                size_t ws_bytes, void* stream, EpLayout* L, Ctx* ctx) {
  switch_status_t s = ep_layout(cfg, ep, L);
  if (s != SWITCH_OK || cfg->T == 0) return s;
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
    return SWITCH_ERR_INVALID_ARG;
  if (ws_bytes < L->total) return SWITCH_ERR_WORKSPACE_TOO_SMALL;
  ctx->C = L->C;
  ctx->ws = static_cast<uint8_t*>(ws);
  ctx->err = reinterpret_cast<DevErr*>(ws);
  ctx->st = static_cast<cudaStream_t>(stream);
  ctx->spin = cfg->spin_limit > 0 ? cfg->spin_limit : kDefaultSpinCycles;
  ctx->num_sms = device_sms();
  if (ctx->num_sms == 0) return SWITCH_ERR_CUDA;
  if (ctx->num_sms < 0) return SWITCH_ERR_UNSUPPORTED;
  return SWITCH_OK;
}

}  // namespace

extern "C" {

int64_t switch_capacity(int64_t T, int32_t n_experts, double capacity_factor) {
  return capacity_exact(T, n_experts, capacity_factor);
}

switch_status_t switch_workspace_size(const switch_config_t* cfg, size_t* bytes) {
  int64_t C = 0;
  switch_status_t s = validate(cfg, &C);
  if (s != SWITCH_OK) return s;
  if (bytes == nullptr) return SWITCH_ERR_INVALID_ARG;
  *bytes = layout_for(*cfg, C).total;
  return SWITCH_OK;
}

switch_status_t switch_backward_workspace_size(const switch_config_t* cfg, size_t* bytes) {
  int64_t C = 0;
  switch_status_t s = validate(cfg, &C);
  if (s != SWITCH_OK) return s;
  if (bytes == nullptr) return SWITCH_ERR_INVALID_ARG;
  *bytes = layout_for(*cfg, C).bwd_total;
  return SWITCH_OK;
}

switch_status_t switch_router(const switch_config_t* cfg, const void* x, const float* w_r,
                              const float* b_r, int32_t* idx, float* gate, float* probs,
                              void* ws, size_t ws_bytes, void* stream) {
  Ctx c{};
  switch_status_t s = prepare(cfg, ws, ws_bytes, stream, &c);
  if (s != SWITCH_OK || cfg->T == 0) return s;
  if (!x || !w_r || !idx || !gate || !aligned16(x) || !aligned16(w_r) ||
      (probs && !aligned16(probs)))
    return SWITCH_ERR_INVALID_ARG;
  const bool top2 = routes_of(*cfg) == 2;
  RouterOut o{idx, gate, probs, c.at<float>(c.L.psum), nullptr, nullptr,
              top2 ? idx + cfg->T : nullptr, top2 ? gate + cfg->T : nullptr};
  if (use_tc_router(cfg)) {
    return cuda_status(launch_router_tc(cfg->T, cfg->d_model, cfg->n_experts,
                                        router_terms(cfg), x, w_r, b_r, c.ws + c.L.wsplit, o,
                                        ntiles_of(cfg->T), c.err, c.spin, c.num_sms, c.st));
  }
  int nparts = 0;
  return cuda_status(launch_router_simt(cfg->T, cfg->d_model, cfg->n_experts,
                                        cfg->dtype == SWITCH_BF16, x, w_r, b_r,
                                        c.at<float>(c.L.logits), o, &nparts, c.st));
}

switch_status_t switch_dispatch(const switch_config_t* cfg, const int32_t* idx,
                                const float* probs, int32_t* rank, uint8_t* drop,
                                int32_t* counts, int32_t* slot_token, const void* x,
                                void* x_disp, void* ws, size_t ws_bytes, void* stream) {
  Ctx c{};
  switch_status_t s = prepare(cfg, ws, ws_bytes, stream, &c);
  if (s != SWITCH_OK || cfg->T == 0) return s;
  if ((!idx && !probs) || !rank || !drop || !counts || !slot_token) return SWITCH_ERR_INVALID_ARG;
  if (x_disp && (!x || !aligned16(x) || !aligned16(x_disp))) return SWITCH_ERR_INVALID_ARG;
  const bool top2 = routes_of(*cfg) == 2;
  if (top2 && !idx) return SWITCH_ERR_INVALID_ARG;      // top-2 dispatch takes the choices
  const int N = cfg->n_experts;
  const int64_t A = routes_of(*cfg) * cfg->T;           // assignments, route-major
  const int nt = ntiles_of(A);
  int* idx_src = idx ? const_cast<int*>(idx) : c.at<int>(c.L.idx);
  SMOE_TRY(launch_tile_rank(A, N, idx, probs, idx ? nullptr : idx_src,
                            c.at<int>(c.L.local_rank), c.at<int>(c.L.hist), nt, c.err, c.st));
  SMOE_TRY(launch_scan(N, nt, c.at<int>(c.L.hist), c.at<int>(c.L.base), counts, c.st));
  if (x_disp) {
    // slots and the row copy in one pass
    const int64_t row_bytes =
        static_cast<int64_t>(cfg->d_model) * (cfg->dtype == SWITCH_BF16 ? 2 : 4);
    SMOE_TRY(launch_finalize_gather(A, N, c.C, nt, idx_src, c.at<int>(c.L.local_rank),
                                    c.at<int>(c.L.base), counts, rank, drop, slot_token,
                                    c.at<int>(c.L.mtile_start), top2 ? cfg->T : 0, x, x_disp,
                                    row_bytes, c.st));
  } else {
    SMOE_TRY(launch_finalize(A, N, c.C, nt, idx_src, c.at<int>(c.L.local_rank),
                             c.at<int>(c.L.base), counts, rank, drop, slot_token,
                             c.at<int>(c.L.mtile_start), top2 ? cfg->T : 0, c.st));
  }
  return SWITCH_OK;
}

switch_status_t switch_expert_ffn(const switch_config_t* cfg, const void* x,
                                  const int32_t* slot_token, const int32_t* counts,
                                  const void* w1, const void* w2, void* y, void* ws,
                                  size_t ws_bytes, void* stream) {
  Ctx c{};
  switch_status_t s = prepare(cfg, ws, ws_bytes, stream, &c);
  if (s != SWITCH_OK || cfg->T == 0) return s;
  const bool dispatched = (cfg->flags & SWITCH_FLAG_ROWS_DISPATCHED) != 0;
  if (!x || (!slot_token && !dispatched) || !counts || !w1 || !w2 || !y || !aligned16(x) ||
      !aligned16(w1) || !aligned16(w2) || !aligned16(y))
    return SWITCH_ERR_INVALID_ARG;
  FfnArgs a{};
  a.T = cfg->T;
  a.d = cfg->d_model;
  a.F = cfg->d_ff;
  a.N = cfg->n_experts;
  a.C = c.C;
  a.x = x;
  a.slot_token = slot_token;
  a.counts = counts;
  a.mtile_start = c.at<int>(c.L.mtile_start);
  a.w1 = w1;
  a.w2 = w2;
  a.hbuf = c.ws + c.L.hbuf;
  a.y = y;
  a.mode2 = kModeY;
  a.err = c.err;
  a.spin = c.spin;
  a.num_sms = c.num_sms;
  a.pair1 = (cfg->flags & SWITCH_FLAG_GEMM_PAIRS) != 0;
  a.pair2 = !(cfg->flags & SWITCH_FLAG_GEMM_1SM);
  a.pair1_rows = gemm1_rows_pairs(cfg, c.C);
  if (dispatched) {
    a.x = nullptr;
    a.x_disp = x;
  }
  if (cfg->dtype == SWITCH_F32) return cuda_status(launch_expert_ffn_f32(a, c.st));
  SMOE_TRY(launch_mtile_table(a.N, a.C, counts, c.at<int>(c.L.mtile_start), c.st));
  if (!dispatched && !(cfg->flags & SWITCH_FLAG_GATHER_IN_GEMM)) {
    SMOE_TRY(launch_gather_rows(static_cast<int64_t>(a.N) * a.C,
                                static_cast<int64_t>(a.d) * 2, slot_token, x,
                                c.ws + c.L.xdisp, c.st));
    a.x_disp = c.ws + c.L.xdisp;
  }
  return cuda_status(launch_expert_ffn_bf16(a, c.st));
}

switch_status_t switch_combine(const switch_config_t* cfg, const void* x_residual,
                               const int32_t* idx, const int32_t* rank, const uint8_t* drop,
                               const float* gate, const void* y, void* out, void* stream) {
  int64_t C = 0;
  switch_status_t s = validate(cfg, &C);
  if (s != SWITCH_OK || cfg->T == 0) return s;
  if (!idx || !rank || !drop || !gate || !y || !out || !aligned16(y) || !aligned16(out) ||
      (x_residual && !aligned16(x_residual)))
    return SWITCH_ERR_INVALID_ARG;
  return cuda_status(launch_combine(cfg->T, cfg->d_model, C, cfg->dtype == SWITCH_BF16,
                                    x_residual, idx, rank, drop, gate, y, out, false,
                                    routes_of(*cfg), static_cast<cudaStream_t>(stream)));
}

switch_status_t switch_aux_loss(const switch_config_t* cfg, const int32_t* counts,
                                const float* probs, float* loss, float* f, float* P, void* ws,
                                size_t ws_bytes, void* stream) {
  Ctx c{};
  switch_status_t s = prepare(cfg, ws, ws_bytes, stream, &c);
  if (s != SWITCH_OK || cfg->T == 0) return s;
  if (!counts || !probs || !loss) return SWITCH_ERR_INVALID_ARG;
  float* psum = c.at<float>(c.L.psum);
  return cuda_status(launch_aux_loss_probs(cfg->T, cfg->n_experts, cfg->alpha, counts, probs,
                                           psum, loss, f, P, c.at<double>(c.L.fpsc),
                                           c.at<unsigned>(kRunTicketOffset),
                                           c.at<unsigned>(kTicketOffset), c.st));
}

switch_status_t switch_layer_forward(const switch_config_t* cfg, const void* x,
                                     const float* w_r, const float* b_r, const void* w1,
                                     const void* w2, void* out, int32_t* idx, float* gate,
                                     int32_t* counts, float* loss, void* ws, size_t ws_bytes,
                                     void* stream) {
  Ctx c{};
  switch_status_t s = prepare(cfg, ws, ws_bytes, stream, &c);
  if (s != SWITCH_OK || cfg->T == 0) return s;
  if (!x || !w_r || !w1 || !w2 || !out || !aligned16(x) || !aligned16(w_r) || !aligned16(w1) ||
      !aligned16(w2) || !aligned16(out))
    return SWITCH_ERR_INVALID_ARG;
  const int64_t T = cfg->T;
  const int N = cfg->n_experts;
  const int nt = ntiles_of(T);
  const bool bf16 = cfg->dtype == SWITCH_BF16;
  const bool top2 = routes_of(*cfg) == 2;
  const int64_t A = routes_of(*cfg) * T;                // assignments, route-major
  const int nta = ntiles_of(A);
  // SWITCH_FLAG_TRAINING: keep probabilities, routing, x_disp and H in the
  // workspace for switch_layer_backward (routing arrays always in the
  // workspace, copied out to the caller's at the end)
  const bool training = (cfg->flags & SWITCH_FLAG_TRAINING) != 0;
  if (training && ws_bytes < c.L.bwd_total) return SWITCH_ERR_WORKSPACE_TOO_SMALL;
  int* idx_p = (idx && !training) ? idx : c.at<int>(c.L.idx);
  float* gate_p = (gate && !training) ? gate : c.at<float>(c.L.gate);
  int* counts_p = (counts && !training) ? counts : c.at<int>(c.L.counts);
  int* local_rank = c.at<int>(c.L.local_rank);
  int* hist = c.at<int>(c.L.hist);
  float* psum = c.at<float>(c.L.psum);
  int nparts = nt;

  // 1. router (+ per-tile ranks and histograms of the first choices on the
  // tensor-core path)
  RouterOut o{idx_p, gate_p, training ? c.at<float>(c.L.probs_s) : nullptr, psum, nullptr,
              nullptr, top2 ? idx_p + T : nullptr, top2 ? gate_p + T : nullptr};
  if (use_tc_router(cfg)) {
    o.hist = hist;
    o.local_rank = local_rank;
    SMOE_TRY(launch_router_tc(T, cfg->d_model, N, router_terms(cfg), x, w_r, b_r,
                              c.ws + c.L.wsplit, o, nt, c.err, c.spin, c.num_sms, c.st));
  } else {
    SMOE_TRY(launch_router_simt(T, cfg->d_model, N, bf16, x, w_r, b_r,
                                c.at<float>(c.L.logits), o, &nparts, c.st));
    SMOE_TRY(launch_tile_rank(T, N, idx_p, nullptr, nullptr, local_rank, hist, nt, c.err,
                              c.st));
  }
  // 2-3. dispatch: scan over tiles, then rank / drop / slots / tile table.
  // Top-2: the first choices' totals are the loss's counts; then the 2T
  // assignments are ranked as one sequence, first choices first.
  // The load-balancing loss (f_i over the first choices) is formed by the
  // scan that counts the first choices.
  const ScanLoss sl{T, nparts, cfg->alpha, psum, loss, c.at<double>(c.L.fpsc),
                    c.at<unsigned>(kTicketOffset)};
  const ScanLoss* slp = loss ? &sl : nullptr;
  if (top2) {
    SMOE_TRY(launch_scan(N, nt, hist, c.at<int>(c.L.base), c.at<int>(c.L.counts1), c.st, slp));
    SMOE_TRY(launch_tile_rank(A, N, idx_p, nullptr, nullptr, local_rank, hist, nta, c.err,
                              c.st));
  }
  SMOE_TRY(launch_scan(N, nta, hist, c.at<int>(c.L.base), counts_p, c.st, top2 ? nullptr : slp));
  int* slot_token = c.at<int>(c.L.slot_token);
  int* rank = c.at<int>(c.L.rank);
  uint8_t* drop = c.at<uint8_t>(c.L.drop);
  // (bf16, default) the routed rows copied expert by expert in the same pass;
  // with the combine fused into the second GEMM (top-1), the dropped tokens'
  // output rows too
  const bool row_copy = bf16 && !(cfg->flags & SWITCH_FLAG_GATHER_IN_GEMM);
  const bool fused = !(cfg->flags & SWITCH_FLAG_UNFUSED_COMBINE) && !top2;
  const bool residual = !(cfg->flags & SWITCH_FLAG_NO_RESIDUAL);
  const bool dropped_in_copy = row_copy && fused;
  if (row_copy)
    SMOE_TRY(launch_finalize_gather(A, N, c.C, nta, idx_p, local_rank, c.at<int>(c.L.base),
                                    counts_p, rank, drop, slot_token,
                                    c.at<int>(c.L.mtile_start), top2 ? T : 0, x,
                                    c.ws + c.L.xdisp, static_cast<int64_t>(cfg->d_model) * 2,
                                    c.st, dropped_in_copy ? out : nullptr, residual,
                                    /*zero_pad=*/training));
  else
    SMOE_TRY(launch_finalize(A, N, c.C, nta, idx_p, local_rank, c.at<int>(c.L.base), counts_p,
                             rank, drop, slot_token, c.at<int>(c.L.mtile_start),
                             top2 ? T : 0, c.st));
  // 4. experts, with the combine fused into the second GEMM unless asked not
  // to (or top-2: two experts write each token, so Y, then one combine)
  const void* x_res = residual ? x : nullptr;
  FfnArgs a{};
  a.T = T;
  a.d = cfg->d_model;
  a.F = cfg->d_ff;
  a.N = N;
  a.C = c.C;
  a.x = x;
  a.slot_token = slot_token;
  a.counts = counts_p;
  a.mtile_start = c.at<int>(c.L.mtile_start);
  a.w1 = w1;
  a.w2 = w2;
  a.hbuf = c.ws + c.L.hbuf;
  a.y = c.ws + c.L.ybuf;
  a.x_res = x_res;
  a.gate = gate_p;
  a.out = out;
  a.mode2 = fused ? kModeCombine : kModeY;
  a.err = c.err;
  a.spin = c.spin;
  a.num_sms = c.num_sms;
  a.pair1 = (cfg->flags & SWITCH_FLAG_GEMM_PAIRS) != 0;
  a.pair2 = !(cfg->flags & SWITCH_FLAG_GEMM_1SM);
  a.pair1_rows = gemm1_rows_pairs(cfg, c.C);
  if (row_copy) a.x_disp = c.ws + c.L.xdisp;
  a.res_by_slot = row_copy;            // the residual rows from the dispatched copy
  SMOE_TRY(bf16 ? launch_expert_ffn_bf16(a, c.st) : launch_expert_ffn_f32(a, c.st));
  // 5. dropped tokens (fused; unless the row copy wrote them) or every token
  // (unfused)
  if (!dropped_in_copy)
    SMOE_TRY(launch_combine(T, cfg->d_model, c.C, bf16, x_res, idx_p, rank, drop, gate_p,
                            c.ws + c.L.ybuf, out, fused, routes_of(*cfg), c.st));
  if (training) {
    if (idx)
      SMOE_TRY(cudaMemcpyAsync(idx, idx_p, sizeof(int) * A, cudaMemcpyDeviceToDevice, c.st));
    if (gate)
      SMOE_TRY(cudaMemcpyAsync(gate, gate_p, sizeof(float) * A, cudaMemcpyDeviceToDevice, c.st));
    if (counts)
      SMOE_TRY(cudaMemcpyAsync(counts, counts_p, sizeof(int) * N, cudaMemcpyDeviceToDevice,
                               c.st));
  }
  return SWITCH_OK;
}

switch_status_t switch_layer_backward(const switch_config_t* cfg, const void* x,
                                      const float* w_r, const float* b_r, const void* w1,
                                      const void* w2, const void* dout, float dloss, void* dx,
                                      float* dw_r, float* db_r, void* dw1, void* dw2,
                                      float* dgate, void* ws, size_t ws_bytes, void* stream) {
  Ctx c{};
  switch_status_t s = prepare(cfg, ws, ws_bytes, stream, &c);
  if (s != SWITCH_OK) return s;
  if (cfg->T == 0) return SWITCH_OK;
  const bool bf16 = cfg->dtype == SWITCH_BF16;
  if (!x || !w_r || !w1 || !w2 || !dout || !dx || !dw_r || !dw1 || !dw2 || !aligned16(x) ||
      !aligned16(w_r) ||
      !aligned16(w1) || !aligned16(w2) || !aligned16(dout) || !aligned16(dx) ||
      !aligned16(dw1) || !aligned16(dw2))
    return SWITCH_ERR_INVALID_ARG;
  if (ws_bytes < c.L.bwd_total) return SWITCH_ERR_WORKSPACE_TOO_SMALL;
  const int64_t T = cfg->T;
  const int N = cfg->n_experts;
  const int d = cfg->d_model, F = cfg->d_ff;
  const int nt = ntiles_of(T);
  const int64_t S = static_cast<int64_t>(N) * c.C;
  // top-2: route-major arrays of A = 2T assignments (entry T + t is token
  // t's second choice); counts1 = the first choices' totals (the loss's f_i)
  const bool top2 = routes_of(*cfg) == 2;
  const int64_t A = routes_of(*cfg) * T;
  const int nta = ntiles_of(A);
  int* idx = c.at<int>(c.L.idx);
  float* gate = c.at<float>(c.L.gate);
  float* probs = c.at<float>(c.L.probs_s);
  int* counts = c.at<int>(c.L.counts);
  int* counts1 = top2 ? c.at<int>(c.L.counts1) : counts;
  int* local_rank = c.at<int>(c.L.local_rank);
  int* hist = c.at<int>(c.L.hist);
  int* rank = c.at<int>(c.L.rank);
  uint8_t* drop = c.at<uint8_t>(c.L.drop);
  int* slot_token = c.at<int>(c.L.slot_token);
  int* mtile_start = c.at<int>(c.L.mtile_start);
  const bool residual = !(cfg->flags & SWITCH_FLAG_NO_RESIDUAL);

  void* x_disp = c.ws + c.L.xdisp;
  void* hbuf = c.ws + c.L.hbuf;
  const bool saved = (cfg->flags & SWITCH_FLAG_TRAINING) != 0;
  if (saved) {
    // 1'. the forward (same flag) left probabilities, routing and H here;
    // only the row copy is missing if it gathered inside GEMM1 (bf16)
    if (bf16 && (cfg->flags & SWITCH_FLAG_GATHER_IN_GEMM))
      SMOE_TRY(launch_gather_rows(S, static_cast<int64_t>(d) * 2, slot_token, x, x_disp, c.st));
  } else {
    // 1. the forward's routing, dispatch and hidden activations, recomputed
    // (same kernels, same results): probabilities, slots, x_disp, H
    RouterOut o{idx, gate, probs, c.at<float>(c.L.psum), nullptr, nullptr,
                top2 ? idx + T : nullptr, top2 ? gate + T : nullptr};
    if (use_tc_router(cfg)) {
      o.hist = hist;
      o.local_rank = local_rank;
      SMOE_TRY(launch_router_tc(T, d, N, router_terms(cfg), x, w_r, b_r, c.ws + c.L.wsplit, o, nt,
                                c.err, c.spin, c.num_sms, c.st));
    } else {
      int nparts = 0;
      SMOE_TRY(launch_router_simt(T, d, N, bf16, x, w_r, b_r, c.at<float>(c.L.logits), o,
                                  &nparts, c.st));
      SMOE_TRY(launch_tile_rank(T, N, idx, nullptr, nullptr, local_rank, hist, nt, c.err, c.st));
    }
    if (top2) {
      // as the forward: first choices' totals, then the 2T assignments ranked
      SMOE_TRY(launch_scan(N, nt, hist, c.at<int>(c.L.base), counts1, c.st));
      SMOE_TRY(launch_tile_rank(A, N, idx, nullptr, nullptr, local_rank, hist, nta, c.err,
                                c.st));
    }
    SMOE_TRY(launch_scan(N, nta, hist, c.at<int>(c.L.base), counts, c.st));
    if (bf16)
      SMOE_TRY(launch_finalize_gather(A, N, c.C, nta, idx, local_rank, c.at<int>(c.L.base),
                                      counts, rank, drop, slot_token, mtile_start, top2 ? T : 0,
                                      x, x_disp, static_cast<int64_t>(d) * 2, c.st));
    else      // fp32: GEMM1 gathers its rows from x
      SMOE_TRY(launch_finalize(A, N, c.C, nta, idx, local_rank, c.at<int>(c.L.base), counts, rank,
                               drop, slot_token, mtile_start, top2 ? T : 0, c.st));
    FfnArgs a{};
    a.T = T;
    a.d = d;
    a.F = F;
    a.N = N;
    a.C = c.C;
    a.x = x;
    a.x_disp = bf16 ? x_disp : nullptr;
    a.slot_token = slot_token;
    a.counts = counts;
    a.mtile_start = mtile_start;
    a.w1 = w1;
    a.w2 = w2;
    a.hbuf = hbuf;
    a.mode2 = kModeY;
    a.pair1 = (cfg->flags & SWITCH_FLAG_GEMM_PAIRS) != 0;
    a.pair1_rows = gemm1_rows_pairs(cfg, c.C);
    a.gemm1_only = true;
    a.err = c.err;
    a.spin = c.spin;
    a.num_sms = c.num_sms;
    SMOE_TRY(bf16 ? launch_expert_ffn_bf16(a, c.st) : launch_expert_ffn_f32(a, c.st));
  }

  const int Np = (N + 63) / 64 * 64;
  float* dh = c.at<float>(c.L.dh);
  int* n_drop = c.at<int>(c.L.n_drop);
  int* drop_list = c.at<int>(c.L.drop_list);
  const double ls = static_cast<double>(dloss) * cfg->alpha * N / (static_cast<double>(T) * T);
  float* dgate_p = dgate ? dgate : c.at<float>(c.L.dgate);
  if (!bf16) {
    // fp32: the expert gradients on CUDA-core tiles, then the router's; dx
    // per token from its slots' rows, the router term and the residual
    BwdF32Args f{};
    f.T = T;
    f.d = d;
    f.F = F;
    f.N = N;
    f.C = c.C;
    f.counts = counts;
    f.slot_token = slot_token;
    f.gate = gate;
    f.idx = idx;
    f.T2 = top2 ? T : 0;
    f.dout = static_cast<const float*>(dout);
    f.x = static_cast<const float*>(x);
    f.w1 = static_cast<const float*>(w1);
    f.w2 = static_cast<const float*>(w2);
    f.h = static_cast<const float*>(hbuf);
    f.dys = c.at<float>(c.L.ybuf);
    f.da = c.at<float>(c.L.da);
    f.dgp = c.at<float>(c.L.dgp);
    f.dw1 = static_cast<float*>(dw1);
    f.dw2 = static_cast<float*>(dw2);
    f.dxs = c.at<float>(c.L.dxs);
    SMOE_TRY(launch_bwd_f32_experts(f, c.st));
    SMOE_TRY(cudaMemsetAsync(n_drop, 0, sizeof(int), c.st));
    const int ntn = bwd_f32_dgp_parts(F);
    if (top2)
      SMOE_TRY(launch_router_bwd_dh_top2(T, N, Np, c.C, ntn, probs, idx, rank, drop, gate, f.dgp,
                                         counts1, static_cast<float>(ls), dh, c.ws + c.L.dhp,
                                         c.ws + c.L.dhs, dgate_p, drop_list, n_drop, c.st));
    else
      SMOE_TRY(launch_router_bwd_dh(T, N, Np, c.C, ntn, probs, idx, rank, drop, gate, f.dgp,
                                    counts, static_cast<float>(ls), dh, c.ws + c.L.dhp,
                                    c.ws + c.L.dhs, dgate_p, drop_list, n_drop, c.st));
    SMOE_TRY(launch_bwd_f32_router(f, routes_of(*cfg), rank, drop, dh, w_r, dw_r, db_r,
                                   static_cast<float*>(dx), residual, c.st));
    return SWITCH_OK;
  }

  // 2. dY = gate * dout per kept slot; dA and the gate-gradient partials;
  // the expert weight gradients
  void* dys = c.ws + c.L.ybuf;
  SMOE_TRY(launch_bwd_gather(c.C, N, d, F, counts, slot_token, gate, idx, top2 ? T : 0, dout,
                             dys, hbuf, c.st));
  BwdFfnArgs b{};
  b.T = T;
  b.d = d;
  b.F = F;
  b.N = N;
  b.C = c.C;
  b.counts = counts;
  b.mtile_start = mtile_start;
  b.slot_token = slot_token;
  b.w1 = w1;
  b.w2 = w2;
  b.x_disp = x_disp;
  b.hbuf = hbuf;
  b.dys = dys;
  b.da = c.ws + c.L.da;
  b.dgp = c.at<float>(c.L.dgp);
  b.dw1 = dw1;
  b.dw2 = dw2;
  b.dout = dout;
  b.dx = dx;
  b.residual = residual;
  b.pair_dw = !(cfg->flags & SWITCH_FLAG_GEMM_1SM);
  b.err = c.err;
  b.spin = c.spin;
  b.num_sms = c.num_sms;
  SMOE_TRY(launch_bwd_dh(b, c.st));
  SMOE_TRY(launch_bwd_dw(b, c.st));

  // 3. router: dh and its bf16 planes, the weight and bias gradients
  SMOE_TRY(cudaMemsetAsync(n_drop, 0, sizeof(int), c.st));
  if (top2)
    SMOE_TRY(launch_router_bwd_dh_top2(T, N, Np, c.C, (F + 255) / 256, probs, idx, rank, drop,
                                       gate, b.dgp, counts1, static_cast<float>(ls), dh,
                                       c.ws + c.L.dhp, c.ws + c.L.dhs, dgate_p, drop_list, n_drop,
                                       c.st));
  else
    SMOE_TRY(launch_router_bwd_dh(T, N, Np, c.C, (F + 255) / 256, probs, idx, rank, drop, gate,
                                  b.dgp, counts, static_cast<float>(ls), dh, c.ws + c.L.dhp,
                                  c.ws + c.L.dhs, dgate_p, drop_list, n_drop, c.st));
  float* colsum = c.at<float>(c.L.colsum);
  if (db_r) SMOE_TRY(launch_prob_colsum(T, N, dh, colsum, c.st));
  SMOE_TRY(launch_router_bwd_dw_tc(T, N, Np, d, c.ws + c.L.dhp, x, c.at<float>(c.L.rpart),
                                   colsum, dw_r, db_r, c.err, c.spin, c.num_sms, c.st));

  // 4. input gradient: kept tokens in the dX GEMM (dA W1_e and dh W_r in one
  // accumulation), dropped ones from the list
  SMOE_TRY(launch_wr_split(N, d, w_r, c.ws + c.L.wrp, c.st));
  b.dhs = c.ws + c.L.dhs;
  b.wrp = c.ws + c.L.wrp;
  b.n_router = N;
  b.n_pad = Np;
  // top-2: the dX GEMM's rows stay per slot (two slots can hold one token)
  // and are added per token, with the residual, afterwards
  if (top2) b.dxs = c.at<float>(c.L.dxs);
  // on operand-swapped CTA pairs unless one-CTA GEMMs are asked for
  SMOE_TRY((cfg->flags & SWITCH_FLAG_GEMM_1SM) ? launch_bwd_dx(b, c.st)
                                               : launch_bwd_dx_pair(b, c.st));
  if (top2)
    SMOE_TRY(launch_bwd_combine_top2(T, d, c.C, idx, rank, drop, b.dxs, dout, dx, residual,
                                     c.st));
  SMOE_TRY(launch_bwd_dropped(T, N, d, drop_list, n_drop, dh, w_r, dout, dx, residual, c.st));
  return SWITCH_OK;
}

switch_status_t switch_ep_sizes(const switch_config_t* cfg, const switch_ep_t* ep,
                                size_t* ws_bytes, size_t* record_bytes, size_t* recv_bytes) {
  EpLayout L{};
  switch_status_t s = ep_layout(cfg, ep, &L);
  if (s != SWITCH_OK) return s;
  if (ws_bytes) *ws_bytes = L.total;
  if (record_bytes) *record_bytes = L.payload_total;
  if (recv_bytes) *recv_bytes = L.recv_total;
  return SWITCH_OK;
}

switch_status_t switch_ep_route(const switch_config_t* cfg, const switch_ep_t* ep, const void* x,
                                const float* w_r, const float* b_r, int32_t* idx, float* gate,
                                void* record, void* ws, size_t ws_bytes, void* stream) {
  EpLayout L{};
  Ctx c{};
  switch_status_t s = ep_prepare_call(cfg, ep, ws, ws_bytes, stream, &L, &c);
  if (s != SWITCH_OK) return s;
  if (cfg->T == 0) return SWITCH_OK;
  if (!record || (reinterpret_cast<uintptr_t>(record) & 15u) != 0 || !x || !w_r ||
      !aligned16(x) || !aligned16(w_r))
    return SWITCH_ERR_INVALID_ARG;
  const int64_t T = cfg->T;
  const int N = cfg->n_experts;
  uint8_t* rec = static_cast<uint8_t*>(record);
  int* idx_w = c.at<int>(L.idx);
  float* gate_w = c.at<float>(L.gate);
  int* hist = c.at<int>(L.hist);
  int* local_rank = c.at<int>(L.local_rank);
  float* psum = reinterpret_cast<float*>(rec);
  SMOE_TRY(cudaMemsetAsync(rec, 0, L.payload_counts, c.st));    // unused parts stay zero
  RouterOut o{idx_w, gate_w, nullptr, psum, nullptr, nullptr, nullptr, nullptr};
  if (L.tc_router) {
    o.hist = hist;
    o.local_rank = local_rank;
    SMOE_TRY(launch_router_tc(T, cfg->d_model, N, router_terms(cfg), x, w_r, b_r,
                              c.ws + L.wsplit, o, L.nt, c.err, c.spin, c.num_sms, c.st));
  } else {
    int nparts = 0;
    SMOE_TRY(launch_router_simt(T, cfg->d_model, N, true, x, w_r, b_r, c.at<float>(L.logits),
                                o, &nparts, c.st));
    SMOE_TRY(launch_tile_rank(T, N, idx_w, nullptr, nullptr, local_rank, hist, L.nt, c.err,
                              c.st));
  }
  SMOE_TRY(launch_scan(N, L.nt, hist, c.at<int>(L.base),
                       reinterpret_cast<int*>(rec + L.payload_counts), c.st));
  if (idx) SMOE_TRY(cudaMemcpyAsync(idx, idx_w, sizeof(int) * T, cudaMemcpyDeviceToDevice, c.st));
  if (gate)
    SMOE_TRY(cudaMemcpyAsync(gate, gate_w, sizeof(float) * T, cudaMemcpyDeviceToDevice, c.st));
  return SWITCH_OK;
}

switch_status_t switch_ep_dispatch(const switch_config_t* cfg, const switch_ep_t* ep,
                                   const void* x, const void* records, void* const* recv_peers,
                                   void* out, int32_t* counts, float* loss, void* ws,
                                   size_t ws_bytes, void* stream) {
  EpLayout L{};
  Ctx c{};
  switch_status_t s = ep_prepare_call(cfg, ep, ws, ws_bytes, stream, &L, &c);
  if (s != SWITCH_OK || cfg->T == 0) return s;
  if (!records || !recv_peers || (reinterpret_cast<uintptr_t>(records) & 15u) != 0)
    return SWITCH_ERR_INVALID_ARG;
  EpPeers peers{};
  for (int i = 0; i < L.G; ++i) {
    if (recv_peers[i] == nullptr || (reinterpret_cast<uintptr_t>(recv_peers[i]) & 255u) != 0)
      return SWITCH_ERR_INVALID_ARG;
    peers.p[i] = recv_peers[i];
  }
  if (!x || !out || !aligned16(x) || !aligned16(out)) return SWITCH_ERR_INVALID_ARG;
  const int N = cfg->n_experts;
  const int64_t T = cfg->T;
  const EpGathered g{static_cast<const uint8_t*>(records), L.payload_total, L.payload_counts};
  int* counts_glob = c.at<int>(L.counts_glob);
  int* counts_loc = c.at<int>(L.counts_loc);
  float* psum_cat = c.at<float>(L.psum_cat);
  SMOE_TRY(launch_ep_prepare(N, L.G, L.r, L.e_loc, L.nparts, g, counts_glob, counts_loc,
                             psum_cat, c.st));
  SMOE_TRY(launch_mtile_table(L.e_loc, L.C, counts_loc, c.at<int>(L.mtile_start), c.st));
  const EpRecvLayout rl{L.recv_src, L.recv_gate};
  int* rank = c.at<int>(L.rank);
  uint8_t* drop = c.at<uint8_t>(L.drop);
  SMOE_TRY(launch_ep_dispatch(T, N, L.C, L.G, L.r, L.e_loc, L.nt, c.at<int>(L.idx),
                              c.at<int>(L.local_rank), c.at<int>(L.base), c.at<float>(L.gate), g,
                              x, static_cast<int64_t>(cfg->d_model) * 2, peers, rl, rank, drop,
                              c.st));
  // dropped tokens: the residual alone, on this rank
  const void* x_res = (cfg->flags & SWITCH_FLAG_NO_RESIDUAL) ? nullptr : x;
  SMOE_TRY(launch_combine(T, cfg->d_model, L.C, true, x_res, c.at<int>(L.idx), rank, drop,
                          c.at<float>(L.gate), nullptr, out, true, 1, c.st));
  if (loss)
    SMOE_TRY(launch_aux_loss(T * L.G, N, L.nparts * L.G, cfg->alpha, counts_glob, psum_cat, loss,
                             nullptr, nullptr, c.at<double>(L.fpsc),
                             c.at<unsigned>(kTicketOffset), c.st));
  if (counts)
    SMOE_TRY(cudaMemcpyAsync(counts, counts_glob, sizeof(int) * N, cudaMemcpyDeviceToDevice,
                             c.st));
  return SWITCH_OK;
}

switch_status_t switch_ep_experts(const switch_config_t* cfg, const switch_ep_t* ep,
                                  const void* w1_local, const void* w2_local, const void* recv,
                                  void* const* out_peers, void* ws, size_t ws_bytes,
                                  void* stream) {
  EpLayout L{};
  Ctx c{};
  switch_status_t s = ep_prepare_call(cfg, ep, ws, ws_bytes, stream, &L, &c);
  if (s != SWITCH_OK || cfg->T == 0) return s;
  if (!w1_local || !w2_local || !recv || !out_peers || !aligned16(w1_local) ||
      !aligned16(w2_local) || (reinterpret_cast<uintptr_t>(recv) & 255u) != 0)
    return SWITCH_ERR_INVALID_ARG;
  for (int i = 0; i < L.G; ++i)
    if (out_peers[i] == nullptr || !aligned16(out_peers[i])) return SWITCH_ERR_INVALID_ARG;
  const uint8_t* rb = static_cast<const uint8_t*>(recv);
  FfnArgs a{};
  a.T = static_cast<int64_t>(L.e_loc) * L.C;
  a.d = cfg->d_model;
  a.F = cfg->d_ff;
  a.N = L.e_loc;
  a.C = L.C;
  a.x = nullptr;
  a.x_disp = rb;
  a.slot_token = reinterpret_cast<const int*>(rb + L.recv_src);
  a.counts = c.at<int>(L.counts_loc);
  a.mtile_start = c.at<int>(L.mtile_start);
  a.w1 = w1_local;
  a.w2 = w2_local;
  a.hbuf = c.ws + L.hbuf;
  a.x_res = (cfg->flags & SWITCH_FLAG_NO_RESIDUAL) ? nullptr : rb;
  a.gate = reinterpret_cast<const float*>(rb + L.recv_gate);
  a.mode2 = kModeCombineEp;
  a.pair1 = (cfg->flags & SWITCH_FLAG_GEMM_PAIRS) != 0;
  a.pair1_rows = gemm1_rows_pairs(cfg, c.C);
  a.pair2 = true;
  a.peer_out = out_peers;
  a.n_peers = L.G;
  a.err = c.err;
  a.spin = c.spin;
  a.num_sms = c.num_sms;
  return cuda_status(launch_expert_ffn_bf16(a, c.st));
}

switch_status_t switch_get_device_error(void* ws, void* stream, int32_t* where_out,
                                        int64_t* info_out) {
  if (ws == nullptr) return SWITCH_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return SWITCH_ERR_CUDA;
  DevErr h{};
  if (cudaMemcpy(&h, ws, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess)
    return SWITCH_ERR_CUDA;
  if (where_out) *where_out = h.where;
  if (info_out) *info_out = h.info;
  if (h.code != 0 && cudaMemset(ws, 0, sizeof(h)) != cudaSuccess) return SWITCH_ERR_CUDA;
  return static_cast<switch_status_t>(h.code);
}

const char* switch_status_string(switch_status_t s) {
  switch (s) {
    case SWITCH_OK: return "ok";
    case SWITCH_ERR_INVALID_ARG: return "invalid argument";
    case SWITCH_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case SWITCH_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case SWITCH_ERR_CUDA: return "CUDA error";
    case SWITCH_ERR_TIMEOUT: return "device wait timed out";
    case SWITCH_ERR_DEVICE_BOUNDS: return "device index out of range";
  }
  return "unknown status";
}

}  // extern "C"
