// Backward pass of the top-1 Switch-FFN layer: parameters of the backward
// GEMM kernel and the launch wrappers the C-ABI layer calls.
#pragma once

#include "kernels.cuh"

namespace smoe {

enum BwdSched : int { kSchedRows = 0, kSchedWeight = 1, kSchedSplit = 2 };
enum BwdEpi : int { kEpiDH = 0, kEpiStore = 1, kEpiDX = 2, kEpiStoreF32 = 3 };

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
  float* out_f32;              // store-f32: [batches * M_out, n_out]
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
  bool residual;
  bool pair_dw;             // weight gradients on CTA pairs (256 x 256 tiles)
  DevErr* err;
  long long spin;
  int num_sms;
};

// dA = (dY W2_e) masked by H > 0, and the per-slot partial gate gradients.
cudaError_t launch_bwd_dh(const BwdFfnArgs& a, cudaStream_t st);
// dW2_e = dY_e^T H_e, dW1_e = dA_e^T X_e for every expert (zeros when empty).
cudaError_t launch_bwd_dw(const BwdFfnArgs& a, cudaStream_t st);
// dx of kept tokens: residual + dA W1_e + dh W_r (the router term as three
// extra bf16 split terms of the same accumulation).
cudaError_t launch_bwd_dx(const BwdFfnArgs& a, cudaStream_t st);
// dW_r [N, d] = dh^T x on the tensor cores: dh as hi + lo bf16 planes
// dhp [2][T][Np] (x is exact in bf16), split-K over token chunks into fp32
// partials `part`, then summed in a fixed order; db [N] (or null) = sum of
// the per-tile column sums colsum [ceil(T / 128)][N].
size_t router_bwd_tc_part_floats(int64_t T, int N, int d, int num_sms);
cudaError_t launch_router_bwd_dw_tc(int64_t T, int N, int Np, int d, const void* dhp,
                                    const void* x, float* part, const float* colsum,
                                    float* dw_r, float* db, DevErr* err, long long spin,
                                    int num_sms, cudaStream_t st);

// dys[s] = bf16(gate[t] * dout[t]) for kept slot s of token t, zero for
// padding; H rows in [kept, min(C, kept rounded up to 64)) of each expert
// are zeroed (the weight-gradient GEMMs read whole 64-row K blocks).
cudaError_t launch_bwd_gather(int64_t C, int N, int d, int F, const int* counts,
                              const int* slot_token, const float* gate, const void* dout,
                              void* dys, void* hbuf, cudaStream_t st);

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
// wrp [2][N][d] = hi / lo bf16 split of W_r (hi = bf16(W), lo = bf16(W - hi)).
cudaError_t launch_wr_split(int N, int d, const float* w_r, void* wrp, cudaStream_t st);
// Dropped tokens (from the list): dx[t] = bf16((residual ? dout[t] : 0) +
// dh[t] . W_r) in fp32.
cudaError_t launch_bwd_dropped(int64_t T, int N, int d, const int* drop_list, const int* n_drop,
                               const float* dh, const float* w_r, const void* dout, void* dx,
                               bool residual, cudaStream_t st);

}  // namespace smoe
