// Backward pass of the top-1 Switch-FFN layer: parameters of the backward
// GEMM kernel and the launch wrappers the C-ABI layer calls.
#pragma once

#include "kernels.cuh"

namespace smoe {

enum BwdSched : int { kSchedRows = 0, kSchedWeight = 1 };
enum BwdEpi : int { kEpiDH = 0, kEpiStore = 1, kEpiDX = 2 };

struct BwdParams {
  int N;                 // experts
  int64_t C;             // capacity
  int M_out;             // weight schedule: output rows per expert
  int n_out;             // output columns
  int K;                 // rows schedule: reduction length (multiple of 64)
  int ntiles_m;          // weight schedule: 128-row tiles per expert
  int ntiles_n;          // 256-column tiles
  int b_rows;            // rows schedule: expert e's B rows start at e * b_rows
  const int* counts;
  const int* mtile_start;
  const int* slot_token;
  const __nv_bfloat16* h;      // dH epilogue: H [N*C, n_out]
  __nv_bfloat16* out;          // dH: dA [N*C, n_out]; store: [N * M_out, n_out]
  float* dgp;                  // dH: [N*C, ntiles_n] partial gate gradients
  const __nv_bfloat16* dout;   // dX: [T, n_out]
  const float* dxr;            // dX: router part of dx [T, n_out]
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
  const float* dxr;         // [T, d] fp32
  void* dx;                 // [T, d] bf16 out (kept tokens)
  bool residual;
  DevErr* err;
  long long spin;
  int num_sms;
};

// dA = (dY W2_e) masked by H > 0, and the per-slot partial gate gradients.
cudaError_t launch_bwd_dh(const BwdFfnArgs& a, cudaStream_t st);
// dW2_e = dY_e^T H_e, dW1_e = dA_e^T X_e for every expert (zeros when empty).
cudaError_t launch_bwd_dw(const BwdFfnArgs& a, cudaStream_t st);
// dx of kept tokens: residual + router part + dA W1_e.
cudaError_t launch_bwd_dx(const BwdFfnArgs& a, cudaStream_t st);

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
cudaError_t launch_router_bwd_dh(int64_t T, int N, int64_t C, int ntn, const float* probs,
                                 const int* idx, const int* rank, const uint8_t* drop,
                                 const float* gate, const float* dgp, const int* counts,
                                 float loss_scale, float* dh, float* dgate, cudaStream_t st);
// dxr [T, d] = dh [T, N] . W_r [N, d]   (fp32 FMA)
cudaError_t launch_router_bwd_dx(int64_t T, int N, int d, const float* dh, const float* w_r,
                                 float* dxr, cudaStream_t st);
// dW_r [N, d] = dh^T x and db [N] = column sums of dh (db may be null), fp32
// FMA, fixed-order split-K over token chunks through `part` (scratch of
// router_bwd_part_floats(T, N, d) floats).
size_t router_bwd_part_floats(int64_t T, int N, int d);
cudaError_t launch_router_bwd_dw(int64_t T, int N, int d, const float* dh, const void* x,
                                 float* part, float* dw_r, float* db, cudaStream_t st);
// Dropped tokens: dx[t] = bf16((residual ? dout[t] : 0) + dxr[t]).
cudaError_t launch_bwd_dropped(int64_t T, int d, const uint8_t* drop, const void* dout,
                               const float* dxr, void* dx, bool residual, cudaStream_t st);

}  // namespace smoe
