// Launch wrappers shared between the kernel files and the C-ABI layer.
#pragma once

#include "common.cuh"

namespace smoe {

constexpr int kTileTok = 128;   // tokens per dispatch/router tile

// ------------------------------------------------------------- dispatch
// Per 128-token tile: expert of each token (from idx, or argmax of probs),
// rank within the tile in token order, and the tile's histogram
// hist[e * ntiles + tile].
cudaError_t launch_tile_rank(int64_t T, int N, const int* idx_in, const float* probs,
                             int* idx_out, int* local_rank, int* hist, int ntiles,
                             DevErr* err, cudaStream_t st);
// The load-balancing loss formed by the scan (as launch_aux_loss would from
// the same counts and per-part sums psum[nparts][N]): fp[N] doubles of
// scratch, ticket one zero-initialised counter (left zero).
struct ScanLoss {
  int64_t T;
  int nparts;
  float alpha;
  const float* psum;
  float* loss;
  double* fp;
  unsigned* ticket;
};
// Exclusive scan of every expert's tile histogram in tile order:
// base[e * ntiles + tile]; counts[e] = total; with `loss`, also the loss
// from these counts.
cudaError_t launch_scan(int N, int ntiles, const int* hist, int* base, int* counts,
                        cudaStream_t st, const ScanLoss* loss = nullptr);
// rank/drop per token, slot_token (kept tokens and -1 padding), and the
// per-expert prefix of 128-row M tiles mtile_start[N + 1].
// tok_mod > 0: entries are route-major assignments of tok_mod tokens, and
// slot_token holds the token (assignment mod tok_mod).
cudaError_t launch_finalize(int64_t T, int N, int64_t C, int ntiles, const int* idx,
                            const int* local_rank, const int* base, const int* counts,
                            int* rank, uint8_t* drop, int* slot_token, int* mtile_start,
                            int64_t tok_mod, cudaStream_t st);
// launch_finalize and the row copy x_disp[slot] = x[token] (zeros in padding
// slots) in one kernel; row_bytes % 16 == 0.  out (top-1 only, tok_mod 0):
// also out[t] = x[t] (out_residual) or zeros for every dropped token t.
// zero_pad false: padding slots are not touched at all, neither their rows
// of x_disp nor their slot_token entries (for a consumer that never reads
// them: the forward GEMMs use only kept slots).
cudaError_t launch_finalize_gather(int64_t T, int N, int64_t C, int ntiles, const int* idx,
                                   const int* local_rank, const int* base, const int* counts,
                                   int* rank, uint8_t* drop, int* slot_token, int* mtile_start,
                                   int64_t tok_mod, const void* x, void* x_disp,
                                   int64_t row_bytes, cudaStream_t st, void* out = nullptr,
                                   bool out_residual = true, bool zero_pad = true);
// Only mtile_start from counts (for a standalone expert-FFN call).
cudaError_t launch_mtile_table(int N, int64_t C, const int* counts, int* mtile_start,
                               cudaStream_t st);
// x_disp[s] = x[slot_token[s]] (zeros for padding), row_bytes % 16 == 0.
cudaError_t launch_gather_rows(int64_t nslots, int64_t row_bytes, const int* slot_token,
                               const void* x, void* x_disp, cudaStream_t st);

// ------------------------------------------------------- combine / loss
// out[t] = x[t] + sum over routes r of (drop ? 0 : gate * y[idx*C + rank]) at
// entry r*T + t; fp32 math, one rounding.  only_dropped (one route): touch
// only dropped tokens (kept ones are written elsewhere).
cudaError_t launch_combine(int64_t T, int d, int64_t C, bool bf16, const void* x,
                           const int* idx, const int* rank, const uint8_t* drop,
                           const float* gate, const void* y, void* out, bool only_dropped,
                           int routes, cudaStream_t st);
// psum[blk][e] = sum of probs rows [blk*128, blk*128 + 128) (fixed order).
cudaError_t launch_prob_colsum(int64_t T, int N, const float* probs, float* psum,
                               cudaStream_t st);
// loss = alpha * N * sum_e (counts_e / T) * (sum_p psum[p][e] / T).
// part_sum: [kAuxChunks][N] doubles; ticket: one zero-initialised counter
// (left zero).
constexpr int kAuxChunks = 16;
cudaError_t launch_aux_loss(int64_t T, int N, int nparts, float alpha, const int* counts,
                            const float* psum, float* loss, float* f, float* P,
                            double* part_sum, unsigned* ticket, cudaStream_t st);

// The loss from full probabilities [T, N] in one launch (column sums per
// 128-row part into psum, then as launch_aux_loss).  run_ticket:
// kAuxChunks zero-initialised counters, ticket: one (all left zero).
cudaError_t launch_aux_loss_probs(int64_t T, int N, float alpha, const int* counts,
                                  const float* probs, float* psum, float* loss, float* f,
                                  float* P, double* part_sum, unsigned* run_ticket,
                                  unsigned* ticket, cudaStream_t st);

// ---------------------------------------------------------------- router
struct RouterOut {
  int* idx;          // [T]
  float* gate;       // [T]
  float* probs;      // [T, N] or null
  float* psum;       // [nparts, N] or null (per-tile sums of probs)
  int* hist;         // [N, ntiles] or null (tensor-core router only)
  int* local_rank;   // [T] or null (tensor-core router only)
  int* idx2;         // top-2: [T] second choices, else null
  float* gate2;      // top-2: [T] their gates
};
// CUDA-core fp32 router; psum parts are 64-token blocks.  `logits` is a
// [T, N] fp32 scratch.
cudaError_t launch_router_simt(int64_t T, int d, int N, bool bf16, const void* x,
                               const float* w_r, const float* b_r, float* logits,
                               RouterOut o, int* nparts_out, cudaStream_t st);
// Tensor-core router (bf16 x).  Writes idx, gate, probs?, psum (128-token
// parts), hist and local_rank.  wsplit: [terms][N_pad][d] bf16 scratch.
cudaError_t launch_router_tc(int64_t T, int d, int N, int terms, const void* x,
                             const float* w_r, const float* b_r, void* wsplit,
                             RouterOut o, int ntiles, DevErr* err, long long spin,
                             int num_sms, cudaStream_t st);
bool router_tc_supported(int N, int d, int terms);
// The CTA-pair router (the one with top-2 support) applies: terms x N_pad <= 256.
bool router_pair_supported(int N, int terms);
// Bytes of the bf16 split-weight scratch launch_router_tc needs (3 terms).
size_t router_wsplit_bytes(int N, int d);

// cuTensorMapEncodeTiled, looked up once through the runtime (expert_ffn.cu).
typedef CUresult (*PFN_encodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                    const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                    const cuuint32_t*, CUtensorMapInterleave,
                                    CUtensorMapSwizzle, CUtensorMapL2promotion,
                                    CUtensorMapFloatOOBfill);
PFN_encodeTiled get_encode_fn();

// 2-D bf16 TMA descriptor (expert_ffn.cu): [outer, inner], box
// box_outer x box_inner, 128-byte swizzle (64-byte when swizzle64).
bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                       uint32_t box_inner, uint32_t box_outer, bool swizzle64 = false);

// ------------------------------------------------------------ expert FFN
// kModeCombineEp: the combine of expert parallelism.  A slot's row of the
// dispatched buffer is its residual, `slot_token` holds the slot's source
// (home rank << kEpRankShift | token on that rank), `gate` is indexed by
// slot, and the output row goes to the home rank's buffer peer_out[rank].
enum GemmMode : int { kModeHidden = 0, kModeY = 1, kModeCombine = 2, kModeCombineEp = 3 };

constexpr int kEpMaxRanks = 16;
constexpr int kEpRankShift = 26;                 // tokens per rank < 2^26

struct FfnArgs {
  int64_t T;
  int d, F, N;
  int64_t C;
  const void* x;            // [T, d]
  const void* x_disp;       // [N*C, d] or null (gather inside GEMM1)
  const int* slot_token;    // [N*C]
  const int* counts;        // [N]
  const int* mtile_start;   // [N + 1]
  const void* w1;           // [N, F, d]
  const void* w2;           // [N, d, F]
  void* hbuf;               // [N*C, F]
  void* y;                  // [N*C, d] (kModeY)
  // kModeCombine: out[token] = x_res[token] + gate[token] * acc
  const void* x_res;        // [T, d] or null
  const float* gate;        // [T]
  void* out;                // [T, d]
  int mode2;                // kModeY or kModeCombine for the second GEMM
  bool pair1;               // GEMM1 on CTA pairs (2-SM), else one CTA per tile
  bool pair2;               // GEMM2 on CTA pairs
  bool pair1_rows;          // GEMM1 on CTA pairs with the rows as M (256-row tiles)
  bool gemm1_only;          // stop after GEMM1 (the backward pass recomputes H)
  // kModeCombine on CTA pairs with x_disp holding every kept row: the
  // residual is read from x_disp by slot (x_res must then be x)
  bool res_by_slot;
  void* const* peer_out;    // kModeCombineEp: every rank's output [T_rank, d] (host array)
  int n_peers;
  DevErr* err;
  long long spin;
  int num_sms;
};
cudaError_t launch_expert_ffn_bf16(const FfnArgs& a, cudaStream_t st);

// ------------------------------------------------------ expert parallelism
// Per-rank exchange record that every rank all-gathers ([G][stride] bytes):
// the per-part router probability sums [nparts][N] fp32 at offset 0 and the
// per-expert token counts [N] int32 at `counts_off`.
struct EpGathered {
  const uint8_t* base;
  size_t stride;
  size_t counts_off;
};
struct EpPeers {
  void* p[kEpMaxRanks];
};
// Receiving rank's buffer: dispatched rows [E_loc*C, d] bf16 at offset 0,
// slot sources [E_loc*C] int32 at src_off, slot gates [E_loc*C] fp32 at
// gate_off.
struct EpRecvLayout {
  size_t src_off;
  size_t gate_off;
};
// Global counts, this rank's experts' counts, and the ranks' probability
// sums laid end to end [G * nparts][N] for the loss.
cudaError_t launch_ep_prepare(int N, int G, int me, int e_loc, int nparts, EpGathered g,
                              int* counts_glob, int* counts_loc, float* psum_cat,
                              cudaStream_t st);
// Global batch-order rank of every token of rank r, drop mask, and the kept
// tokens' rows, sources and gates stored into their owners' buffers.
cudaError_t launch_ep_dispatch(int64_t T, int N, int64_t C, int G, int r, int e_loc, int ntiles,
                               const int* idx, const int* local_rank, const int* base,
                               const float* gate, EpGathered g, const void* x, int64_t row_bytes,
                               const EpPeers& recv, EpRecvLayout rl, int* rank, uint8_t* drop,
                               cudaStream_t st);
cudaError_t launch_expert_ffn_f32(const FfnArgs& a, cudaStream_t st);

}  // namespace smoe
