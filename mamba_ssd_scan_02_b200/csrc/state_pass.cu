// state_pass.cu -- inter-segment state pass of the segmented chunked scan.
//
// When a sequence is split into n_seg segments scanned in parallel, each segment k first
// produces its local final state s_k (scanned from a zero state) and its total decay
// lambda_k = exp(sum of dt*A over the segment).  The state entering segment k is then
//   h_in[0] = h0,   h_in[k] = lambda_{k-1} h_in[k-1] + s_{k-1},
// and the state after the last segment is lambda_{n-1} h_in[n-1] + s_{n-1} = h_final.
// This is the same linear recurrence as the token scan, applied at segment granularity.  The
// same pass joins the spans of a sequence split across GPUs (sequence parallelism): each rank
// scans its span from a zero state, the (s_k, lambda_k) of all spans are gathered, and every
// rank forms the state entering its own span with this recurrence.
// One thread per 4 state elements (float4), sequential over the segments; h_in[k]
// overwrites s_k in place (s_k is read first).  Within a segment the state never leaves the
// scan CTA (it stays in tensor memory from chunk to chunk), so this pass only joins segments:
// a few float4 streams of 4 MiB each, bound by memory, with no data shared between threads.
#include "common.cuh"
#include "plan.h"

namespace ssd {
namespace {

__global__ void state_pass_kernel(const float4 *seg_state, float4 *h_in,
                                  const float *__restrict__ seg_decay, const float4 *__restrict__ h0,
                                  float4 *__restrict__ h_final, float *__restrict__ decay_total,
                                  int n_seg, long long BH, int PN4) {
  // seg_state and h_in may be the same buffer: each slot is read before it is written, by the
  // same thread
  const long long n = BH * PN4;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const long long bh = i / PN4;
    float4 h = h0 ? h0[i] : make_float4(0.f, 0.f, 0.f, 0.f);
    float dec = 1.f;
    for (int k = 0; k < n_seg; ++k) {
      const long long slot = (long long)k * BH * PN4 + i;
      const float4 s = seg_state[slot];
      if (h_in) h_in[slot] = h;
      const float a = seg_decay[(long long)k * BH + bh];
      h = make_float4(a * h.x + s.x, a * h.y + s.y, a * h.z + s.z, a * h.w + s.w);
      dec *= a;
    }
    if (h_final) h_final[i] = h;
    if (decay_total && i % PN4 == 0) decay_total[bh] = dec;
  }
}

// The final state's fold after the tail pass: h = dec h + dh per (batch row, head), where
// dh and dec are what the last chunks contribute from a zero state and their total decay.
__global__ void tail_fold_kernel(float4 *__restrict__ h, const float4 *__restrict__ dh,
                                 const float *__restrict__ dec, long long n4, long long h4_extent, int *err) {
  constexpr int kPer = kHeadDim * kDState / 4;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (long long)gridDim.x * blockDim.x) {
    const float d = dec[i / kPer];
    float4 v = h[i];
    const float4 a = dh[i];
    v.x = fmaf(d, v.x, a.x); v.y = fmaf(d, v.y, a.y); v.z = fmaf(d, v.z, a.z); v.w = fmaf(d, v.w, a.w);
    if (in_bounds(i, h4_extent, err)) h[i] = v;
  }
}

}  // namespace

cudaError_t launch_tail_fold(const PrefillPlan &p, cudaStream_t s) {
  if (!p.tail_dh || p.L == 0) return cudaSuccess;
  const long long n4 = (long long)p.B * p.H * kHeadDim * kDState / 4;
  long long blocks = (n4 + 255) / 256;
  if (blocks > 148 * 8) blocks = 148 * 8;
  tail_fold_kernel<<<(unsigned)blocks, 256, 0, s>>>(reinterpret_cast<float4 *>(p.h_final),
                                                     reinterpret_cast<const float4 *>(p.tail_dh), p.tail_dec, n4,
                                                     checked_extent(p, n4), p.err);
  return cudaGetLastError();
}

cudaError_t launch_span_prefix(const float *states, float *h_in, const float *decays, int n_spans,
                               long long BH, int PN, const float *h0, float *h_final,
                               float *decay_total, cudaStream_t s) {
  const int PN4 = PN / 4;
  const long long n = BH * PN4;
  if (n == 0) return cudaSuccess;
  long long g = (n + 255) / 256;
  if (g > 148 * 8) g = 148 * 8;
  state_pass_kernel<<<(int)g, 256, 0, s>>>(reinterpret_cast<const float4 *>(states),
                                           reinterpret_cast<float4 *>(h_in), decays,
                                           reinterpret_cast<const float4 *>(h0),
                                           reinterpret_cast<float4 *>(h_final), decay_total,
                                           n_spans, BH, PN4);
  return cudaGetLastError();
}

cudaError_t launch_state_pass(const PrefillPlan &p, cudaStream_t s) {
  return launch_span_prefix(p.seg_state, p.seg_state, p.seg_decay, p.n_seg, (long long)p.B * p.H,
                            p.P * p.N, p.h0, p.h_final, nullptr, s);
}

}  // namespace ssd
