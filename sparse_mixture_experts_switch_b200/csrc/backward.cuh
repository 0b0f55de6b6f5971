// Backward pass of the Switch-FFN layer (top-1 and top-2): parameters of the backward
// GEMM kernel and the launch wrappers the C-ABI layer calls.
#pragma once

#include "kernels.cuh"

namespace smoe {

enum BwdSched : int { kSchedRows = 0, kSchedWeight = 1, kSchedSplit = 2 };
enum BwdEpi : int { kEpiDH = 0, kEpiStore = 1, kEpiDX = 2, kEpiStoreF32 = 3, kEpiDXSlot = 4 };

struct BwdParams {
  int N;                 // experts
  int64_t C;             // capacity
  int M_out;             // weight schedule: output rows per expert
  int n_out;             // output columns
  int K;                 // rows schedule: reduction length (multiple of 64)
  int ntiles_m;          // weight schedule: 128-row tiles per expert
  int ntiles_n;          // 256-column tiles
  int b_rows;            // rows schedule: expert e's B rows start at e * b_rows
  int kx_blocks;         // rows schedule: extra K blocks per extra term (router term of dX)
  int kx_terms;          //   extra terms (0: none; 3: hi.hi + lo.hi + hi.lo)
  int nsplit;            // split schedule: K chunks per term
  int64_t split_len;     //   rows per chunk (multiple of 64)
  int64_t split_rows;    //   total K rows (T)
  const int* counts;
  const int* mtile_start;
  const int* slot_token;
  const __nv_bfloat16* h;      // dH epilogue: H [N*C, n_out]
  __nv_bfloat16* out;          // dH: dA [N*C, n_out]; store: [N * M_out, n_out]
  float* out_f32;              // store-f32: [batches * M_out, n_out]; dX per slot: [N*C, n_out]
  float* dgp;                  // dH: [N*C, ntiles_n] partial gate gradients
  const __nv_bfloat16* dout;   // dX: [T, n_out]
  __nv_bfloat16* dx;           // dX: [T, n_out]
  int residual;                // dX: add dout (the residual branch)
  DevErr* err;
  long long spin;
};

struct BwdFfnArgs {
  int64_t T;
  int d, F, N;
  int64_t C;
  const int* counts;        // [N]
  const int* mtile_start;   // [N + 1]
  const int* slot_token;    // [N*C]
  const void* w1;           // [N, F, d] bf16
  const void* w2;           // [N, d, F] bf16
  const void* x_disp;       // [N*C, d] bf16, zero padding rows
  const void* hbuf;         // [N*C, F] bf16 (H; padding rows zeroed to the K block)
  const void* dys;          // [N*C, d] bf16: gate * dout of each kept slot, zero padding
  void* da;                 // [N*C, F] bf16 out
  float* dgp;               // [N*C, ceil(F / 256)] out
  void* dw1;                // [N, F, d] bf16 out
  void* dw2;                // [N, d, F] bf16 out
  const void* dout;         // [T, d] bf16
  const void* dhs;          // [2][N*C][Np] bf16: hi / lo planes of dh per kept slot
  const void* wrp;          // [2][N][d] bf16: hi / lo planes of W_r
  int n_router, n_pad;      // router experts N and the planes' row length Np
  void* dx;                 // [T, d] bf16 out (kept tokens)
  float* dxs;               // top-2: [N*C, d] fp32 out, the dX GEMM's rows per kept slot
                            // (then added per token by launch_bwd_combine_top2); null: top-1
  bool residual;
  bool pair_dw;             // weight gradients on CTA pairs (256 x 256 tiles)
  DevErr* err;
  long long spin;
  int num_sms;
};

// dA = (dY W2_e) masked by H > 0, and the per-slot partial gate gradients.
cudaError_t launch_bwd_dh(const BwdFfnArgs& a, cudaStream_t st);
// 3-D bf16 TMA descriptor [outer][mid][inner], box 1 x box_mid x box_inner,
// 128-byte swizzle (backward_gemm.cu).
bool make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t mid,
                       uint64_t outer, uint32_t box_inner, uint32_t box_mid);
// dW2_e = dY_e^T H_e, dW1_e = dA_e^T X_e for every expert (zeros when empty).
cudaError_t launch_bwd_dw(const BwdFfnArgs& a, cudaStream_t st);
// dx of kept tokens: residual + dA W1_e + dh W_r (the router term as three
// extra bf16 split terms of the same accumulation).  With a.dxs (top-2: two
// slots may hold one token) each kept slot's fp32 row dA W1_e + dh_s W_r is
// stored at its slot instead, without the residual.
cudaError_t launch_bwd_dx(const BwdFfnArgs& a, cudaStream_t st);
// The same on operand-swapped CTA pairs (output features x slots per tile,
// slots as the MMA's flexible N; backward_pair.cu).
cudaError_t launch_bwd_dx_pair(const BwdFfnArgs& a, cudaStream_t st);
// dW_r [N, d] = dh^T x on the tensor cores: dh as hi + lo bf16 planes
// dhp [2][T][Np] (x is exact in bf16), split-K over token chunks into fp32
// partials `part`, then summed in a fixed order; db [N] (or null) = sum of
// the per-tile column sums colsum [ceil(T / 128)][N].
size_t router_bwd_tc_part_floats(int64_t T, int N, int d, int num_sms);
cudaError_t launch_router_bwd_dw_tc(int64_t T, int N, int Np, int d, const void* dhp,
                                    const void* x, float* part, const float* colsum,
                                    float* dw_r, float* db, DevErr* err, long long spin,
                                    int num_sms, cudaStream_t st);

// dys[s] = bf16(g * dout[t]) for kept slot s of token t, zero for padding;
// g = gate[t] (top-1), or with top-2 (T2 = T > 0) the gate of the route that
// put t in expert e = s / C: gate[t] if idx[t] == e (its first choice), else
// gate[T2 + t].  H rows in [kept, min(C, kept rounded up to 64)) of each
// expert are zeroed (the weight-gradient GEMMs read whole 64-row K blocks).
cudaError_t launch_bwd_gather(int64_t C, int N, int d, int F, const int* counts,
                              const int* slot_token, const float* gate, const int* idx,
                              int64_t T2, const void* dout, void* dys, void* hbuf,
                              cudaStream_t st);

// Router backward for top-1 routing:
//   dgate[t] = sum_j dgp[idx*C + rank][j] / gate[t] (kept tokens, else 0),
//   dp[t, i] = loss_scale * counts[i] + [i == idx, kept] dgate[t],
//   dh[t, i] = p[t, i] (dp[t, i] - sum_j p[t, j] dp[t, j]).
// loss_scale = dloss * alpha * N / T^2 (the load-balancing loss's gradient
// per routed token).
// Outputs: dh [T, N] fp32 (probs is left as it is), its hi / lo bf16 planes
// dhp [2][T][Np] and, for kept tokens, dhs [2][N*C][Np] at the token's slot
// (columns N..Np-1 zero), the gate gradient, and the list of dropped tokens
// (drop_list[0..*n_drop), any order; *n_drop must be zero on entry).
cudaError_t launch_router_bwd_dh(int64_t T, int N, int Np, int64_t C, int ntn,
                                 const float* probs, const int* idx, const int* rank,
                                 const uint8_t* drop, const float* gate, const float* dgp,
                                 const int* counts, float loss_scale, float* dh, void* dhp,
                                 void* dhs, float* dgate, int* drop_list, int* n_drop,
                                 cudaStream_t st);
// Router backward for top-2 routing: per token t and route r (entry
// a = r T + t of the route-major arrays idx, rank, drop, gate, dgate),
//   dgate[a] = sum_j dgp[idx_a*C + rank_a][j] / gate[a] (kept route, gate > 0;
//              else 0),
//   dp[t, i] = loss_scale * counts1[i] + sum over kept r with idx_a = i of dgate[a],
//   dh[t, i] = p[t, i] (dp[t, i] - sum_j p[t, j] dp[t, j]);
// counts1 are the first choices' totals (the loss's f_i).  dh's hi / lo
// planes go to dhp [2][T][Np], and to dhs [2][N*C][Np] at the token's first
// kept slot (route 0 if kept, else route 1); a second kept slot gets zero
// planes, so the router term dh W_r enters the token's dx once.  Tokens with
// both routes dropped are listed in drop_list (any order).
cudaError_t launch_router_bwd_dh_top2(int64_t T, int N, int Np, int64_t C, int ntn,
                                      const float* probs, const int* idx, const int* rank,
                                      const uint8_t* drop, const float* gate, const float* dgp,
                                      const int* counts1, float loss_scale, float* dh,
                                      void* dhp, void* dhs, float* dgate, int* drop_list,
                                      int* n_drop, cudaStream_t st);
// Top-2 input gradient of tokens with at least one kept route:
//   dx[t] = bf16((residual ? dout[t] : 0) + dxs[s_0] + dxs[s_1])  (kept routes'
// slots s_r = idx_a*C + rank_a, added in route order in fp32).  Tokens with
// both routes dropped are left to launch_bwd_dropped.
cudaError_t launch_bwd_combine_top2(int64_t T, int d, int64_t C, const int* idx, const int* rank,
                                    const uint8_t* drop, const float* dxs, const void* dout,
                                    void* dx, bool residual, cudaStream_t st);
// ------------------------------------------------------------ fp32 path
// The backward in fp32 on CUDA-core FMA tiles (backward_f32.cu).
struct BwdF32Args {
  int64_t T;
  int d, F, N;
  int64_t C;
  const int* counts;        // [N]
  const int* slot_token;    // [N*C]
  const float* gate;        // [routes * T]
  const int* idx;           // [routes * T]
  int64_t T2;               // top-2: T (a slot's route from idx), else 0
  const float* dout;        // [T, d]
  const float* x;           // [T, d]
  const float* w1;          // [N, F, d]
  const float* w2;          // [N, d, F]
  const float* h;           // [N*C, F] hidden activations of the forward
  float* dys;               // [N*C, d] out: gate * dout per kept slot
  float* da;                // [N*C, F] out
  float* dgp;               // [N*C, bwd_f32_dgp_parts(F)] out
  float* dw1;               // [N, F, d] out
  float* dw2;               // [N, d, F] out
  float* dxs;               // [N*C, d] out: dA W1_e per kept slot
};
// Gate-gradient partials per slot of the fp32 dH (one per 64 columns).
int bwd_f32_dgp_parts(int F);
// dY, dA and its gate-gradient partials, dW2, dW1 and the dX rows per slot.
cudaError_t launch_bwd_f32_experts(const BwdF32Args& a, cudaStream_t st);
// dW_r = dh^T x, db_r = column sums of dh (if db_r), and
// dx[t] = residual + the token's kept slots' dX rows + dh[t] W_r.
cudaError_t launch_bwd_f32_router(const BwdF32Args& a, int routes, const int* rank,
                                  const uint8_t* drop, const float* dh, const float* w_r,
                                  float* dw_r, float* db_r, float* dx, bool residual,
                                  cudaStream_t st);

// wrp [2][N][d] = hi / lo bf16 split of W_r (hi = bf16(W), lo = bf16(W - hi)).
cudaError_t launch_wr_split(int N, int d, const float* w_r, void* wrp, cudaStream_t st);
// Dropped tokens (from the list): dx[t] = bf16((residual ? dout[t] : 0) +
// dh[t] . W_r) in fp32.
cudaError_t launch_bwd_dropped(int64_t T, int N, int d, const int* drop_list, const int* n_drop,
                               const float* dh, const float* w_r, const void* dout, void* dx,
                               bool residual, cudaStream_t st);

}  // namespace smoe
