// plan.h -- resolved launch parameters shared by the C-ABI layer and the kernel launchers.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>

#include "../../include/ssd.h"

namespace ssd {

// Everything a prefill launch needs, after validation: shapes, pointers, workspace carve-outs.
struct PrefillPlan {
  int B, L, H, P, N, G, Q, W, norm_groups;
  // Variable-length batch (tensor path): the B sequences are packed back to back, sequence b
  // being rows cu[b] .. cu[b+1]-1 of every token tensor (cu: device, B + 1 offsets), and L is
  // the longest length; null for a uniform batch (row b*L + t).  rows = the number of token
  // rows (B*L, or cu[B]).
  const int *cu;
  long long rows;
  int nbg;           // 1: normalise before gating (out = rmsnorm(y) * w * silu(z))
  int hpg, d_inner, conv_dim;
  float eps, dt_min, dt_max;
  int softplus;
  bool bf16;
  int n_seg, seg_len;  // internal sequence segments (1 = none)
  // user tensors
  const void *xBC; long long xs;
  const void *dt;  long long ds;
  const void *z;   long long zs;
  const float *A, *D, *dt_bias;
  const void *conv_w, *conv_b, *norm_w;
  const float *h0;
  const void *csi;
  void *y; long long ys;
  float *h_final;
  void *cso;
  // workspace
  float *u;          // [B, L, conv_dim] conv+SiLU output (SIMT path)
  float *dte;        // [B, L, H] effective dt
  float *yf;         // [B, L, d_inner] pre-norm output (when norm_groups > 0)
  float *seg_state;  // [n_seg, B, H, P, N]
  float *seg_decay;  // [n_seg, B, H]
  void *bc;          // [B, L, 2*G*N] fp16 conv+SiLU output of the B|C channels (tensor path)
  float *dte_hm;     // [B, H, Lpad] effective dt, head-major (tensor path)
  float *cs_hm;      // [B, H, Lpad] chunk-local prefix sums of dt*A (tensor path)
  float *tail_dh;    // [B, H, P, N] fp32 contribution of the final state's last chunks, from a
                     // zero state (tensor path; null when no final state is written)
  float *tail_dec;   // [B, H] decay over those chunks
  __half *yh;        // [rows, d_inner] fp16 pre-norm output (tensor path, when the gated
                     // norm follows: its pass reads y with z)
  int Lpad;
  int *err;          // device error word
  // test hook (tensor-core scan): 0 = off; c + 1 = the producer withholds chunk c's stage so
  // that the bounded waits run out after stall_wait_ns
  int stall_chunk1;
  unsigned long long stall_wait_ns;
  // test hook of the debug build's index checks: the extents they allow are the buffers'
  // divided by this (1 = the buffers' own)
  int bounds_denom;
};

// The extent (elements) the index checks of the debug build allow for a buffer of n elements.
inline long long checked_extent(const PrefillPlan &p, long long n) {
  return p.bounds_denom > 1 ? n / p.bounds_denom : n;
}

struct DecodePlan {
  int B, H, P, N, G, W, norm_groups, hpg, d_inner, conv_dim;
  int nbg;           // 1: normalise before gating
  float eps, dt_min, dt_max;
  int softplus;
  bool bf16;
  const void *xBC; long long xs;
  const void *dt;  long long ds;
  const void *z;   long long zs;
  const float *A, *D, *dt_bias;
  const void *conv_w, *conv_b, *norm_w;
  float *state;
  const void *csi;
  void *cso;
  void *y; long long ys;
};

// front end (frontend.cu)
cudaError_t launch_conv_silu_f32(const PrefillPlan &p, cudaStream_t s);
cudaError_t launch_dt(const PrefillPlan &p, cudaStream_t s);
cudaError_t launch_conv_state_out(const PrefillPlan &p, cudaStream_t s);
cudaError_t launch_carry_only(const PrefillPlan &p, cudaStream_t s);  // seqlen == 0
cudaError_t launch_bc_conv_f16(const PrefillPlan &p, cudaStream_t s);
// dt + prefix sums, B/C conv and (if with_cso) the outgoing conv cache in one launch
bool front_tc_fusable(const PrefillPlan &p);
cudaError_t launch_front_tc(const PrefillPlan &p, bool with_cso, cudaStream_t s);  // B|C channels -> p.bc (fp16)
cudaError_t launch_dt_cumsum(const PrefillPlan &p, float *dte, float *cs, int Lpad, cudaStream_t s);
// chunked scan on CUDA cores (scan_simt.cu); mode 0 full, 1 state-only, 2 output-only
cudaError_t launch_scan_simt(const PrefillPlan &p, int mode, cudaStream_t s);
// chunked scan on tcgen05 tensor cores (tc_scan.cu); mode 0 full/output, 1 state-only
bool tc_scan_available();
cudaError_t launch_scan_tc(const PrefillPlan &p, int mode, cudaStream_t s);
// inter-segment state pass (state_pass.cu)
cudaError_t launch_state_pass(const PrefillPlan &p, cudaStream_t s);
// The same linear recurrence over spans held elsewhere (sequence parallelism): h_in[k] (may be
// `states` itself, in place) = the state entering span k; h_final and decay_total optional.
cudaError_t launch_span_prefix(const float *states, float *h_in, const float *decays, int n_spans,
                               long long BH, int PN, const float *h0, float *h_final,
                               float *decay_total, cudaStream_t s);
// fp32 recomputation of the final state's last kTailChunks chunks (tensor-core path): what
// those chunks add to a zero state, into p.tail_dh / p.tail_dec.  It runs on a side stream
// beside the output scan, which leaves the state entering those chunks in h_final; the fold
// then sets h_final = tail_dec * h_final + tail_dh.
constexpr int kTailChunks = 2;
// Where the tail pass runs: beside the output scan (on a side stream, on the SMs the scan
// leaves free) when those SMs finish all its items within the scan's time; otherwise after the
// scan on the same stream, where it folds into h_final itself (fold_in: no dH, no fold pass).
bool tail_beside_scan(const PrefillPlan &p);
cudaError_t launch_state_tail(const PrefillPlan &p, bool fold_in, cudaStream_t s);
cudaError_t launch_tail_fold(const PrefillPlan &p, cudaStream_t s);
// norms (norm.cu)
cudaError_t launch_gated_norm(const PrefillPlan &p, cudaStream_t s);  // yh (fp16) or yf (fp32) -> y
// RMSNorm folded into the projection that follows it: r[row] = 1 / sqrt(mean(x[row]^2) + eps)
// (fp32), and W'[n][k] = W[n][k] * w[k] (bf16), so that rmsnorm(x) W^T = diag(r) x W'^T.
cudaError_t launch_rms_rowscale_bf16(const void *x, float *r, long long rows, int width, float eps,
                                     cudaStream_t s);
cudaError_t launch_fold_cols_bf16(const void *W, const void *w, void *out, long long rows, int K,
                                  cudaStream_t s);
// decode (decode.cu)
cudaError_t launch_decode(const DecodePlan &p, cudaStream_t s);
// GEMM C[M,N] = diag(row_scale) A[M,K] . B[N,K]^T, bf16 in/out, fp32 accumulate (row_scale:
// fp32 [M] or null for none)
cudaError_t launch_gemm_bf16_tn(const void *A, long long lda, const void *Bm, long long ldb, void *C,
                                long long ldc, int M, int N, int K, cudaStream_t s,
                                const float *row_scale = nullptr);
cudaError_t launch_gemm_tc_bf16_tn(const void *A, long long lda, const void *Bm, long long ldb, void *C,
                                   long long ldc, int M, int N, int K, int *err, cudaStream_t s,
                                   const float *row_scale = nullptr);
cudaError_t launch_gemm_simt_bf16_tn(const void *A, long long lda, const void *Bm, long long ldb,
                                     void *C, long long ldc, int M, int N, int K, cudaStream_t s,
                                     const float *row_scale = nullptr);

// ---- tracing (trace.cu): event pairs around each launch while enabled ------------------
bool trace_enabled();
int trace_begin(cudaStream_t s);                        // -1 when tracing is off
void trace_end(int slot, const char *name, cudaStream_t s);

template <class F>
cudaError_t traced(const char *name, cudaStream_t s, F &&launch) {
  const int slot = trace_begin(s);
  cudaError_t e = launch();
  if (slot >= 0) trace_end(slot, name, s);
  return e;
}

}  // namespace ssd
