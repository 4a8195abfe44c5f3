// state_tail.cu -- the final state's last chunks in fp32.
//
// The tensor-core scan carries the state in fp32 but multiplies fp16 operands, and the final
// state's largest entries often come from a few recent tokens, whose products are not
// averaged over many terms.  So the scan leaves the state entering the last kTailChunks
// chunks of the sequence (of its last segment), and this pass finishes the recurrence over
// those chunks from the raw inputs in fp32:
//   per chunk:  h <- e^{cs_Q} h + sum_s e^{cs_Q - cs_s} dt_s x_s B_s^T
// with x_s, B_s the causal conv1d + SiLU of the raw channels (history from the incoming conv
// cache before token 0) and dt_s, cs_s the chunk-local prefix sums of dt*A already computed
// for the scan.  One CTA per (head, batch row); thread t owns state row p = t / 4 and
// columns 32 (t % 4) .. +31; conv outputs are staged in shared memory 32 tokens at a time.
#include "common.cuh"
#include "plan.h"

namespace ssd {
namespace {

constexpr int kTailThreads = 256;
constexpr int kTailTok = 32;

__global__ void __launch_bounds__(kTailThreads) state_tail_kernel(
    const __nv_bfloat16 *__restrict__ xBC, long long xs, const __nv_bfloat16 *__restrict__ conv_w,
    const __nv_bfloat16 *__restrict__ conv_b, const __nv_bfloat16 *__restrict__ csi,
    const float *__restrict__ dte, const float *__restrict__ cs, float *__restrict__ hstate, int L,
    int H, int hpg, int conv_dim, int d_inner, int W, int Lpad, int t_tail) {
  __shared__ __align__(16) float ux[kTailTok][kHeadDim];
  __shared__ __align__(16) float uB[kTailTok][kDState];
  __shared__ float ws[kTailTok];
  const int h = blockIdx.x, b = blockIdx.y, g = h / hpg;
  const int tid = threadIdx.x, p = tid >> 2, n0 = (tid & 3) * 32;
  float *hrow = hstate + (((long long)b * H + h) * kHeadDim + p) * kDState + n0;
  float acc[32];
#pragma unroll
  for (int j = 0; j < 32; j += 4) {
    const float4 v = *reinterpret_cast<const float4 *>(hrow + j);
    acc[j] = v.x; acc[j + 1] = v.y; acc[j + 2] = v.z; acc[j + 3] = v.w;
  }
  const float *csr = cs + ((long long)b * H + h) * Lpad;
  const float *dtr = dte + ((long long)b * H + h) * Lpad;
  const __nv_bfloat16 *xrow = xBC + (long long)b * L * xs;
  for (int c0 = t_tail; c0 < L; c0 += 128) {
    const float csQ = csr[c0 + 127];  // the padding past L has dt = 0: the prefix stays flat
    const float decay = __expf(csQ);
#pragma unroll
    for (int j = 0; j < 32; ++j) acc[j] *= decay;
    const int cend = min(c0 + 128, L);
    for (int s0 = c0; s0 < cend; s0 += kTailTok) {
      __syncthreads();  // the previous block's conv outputs are consumed
      for (int idx = tid; idx < kTailTok * (kHeadDim + kDState); idx += kTailThreads) {
        const int s = idx / (kHeadDim + kDState), ch = idx % (kHeadDim + kDState), t = s0 + s;
        const int c = ch < kHeadDim ? h * kHeadDim + ch : d_inner + g * kDState + (ch - kHeadDim);
        float v = 0.f;
        if (t < cend) {
          if (W == 0) {
            v = __bfloat162float(xrow[(long long)t * xs + c]);
          } else {
            float u = conv_b ? __bfloat162float(conv_b[c]) : 0.f;
            for (int k = 0; k < W; ++k) {  // tap k multiplies time t - (W-1) + k
              const int tau = t - (W - 1) + k;
              float xv = 0.f;
              if (tau >= 0) xv = __bfloat162float(xrow[(long long)tau * xs + c]);
              else if (csi && W + tau >= 0) xv = __bfloat162float(csi[((long long)b * W + (W + tau)) * conv_dim + c]);
              u = fmaf(__bfloat162float(conv_w[(long long)c * W + k]), xv, u);
            }
            v = silu(u);
          }
        }
        if (ch < kHeadDim) ux[s][ch] = v;
        else uB[s][ch - kHeadDim] = v;
      }
      if (tid < kTailTok) {
        const int t = s0 + tid;
        ws[tid] = t < cend ? __expf(csQ - csr[t]) * dtr[t] : 0.f;
      }
      __syncthreads();
      for (int s = 0; s < kTailTok; ++s) {
        const float aw = ws[s] * ux[s][p];
        const float2 aw2 = make_float2(aw, aw);
        const float4 *bq = reinterpret_cast<const float4 *>(&uB[s][n0]);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 v = bq[q];
          const float2 lo = __ffma2_rn(aw2, make_float2(v.x, v.y), make_float2(acc[4 * q], acc[4 * q + 1]));
          const float2 hi = __ffma2_rn(aw2, make_float2(v.z, v.w), make_float2(acc[4 * q + 2], acc[4 * q + 3]));
          acc[4 * q] = lo.x; acc[4 * q + 1] = lo.y; acc[4 * q + 2] = hi.x; acc[4 * q + 3] = hi.y;
        }
      }
    }
  }
#pragma unroll
  for (int j = 0; j < 32; j += 4)
    *reinterpret_cast<float4 *>(hrow + j) = make_float4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]);
}

}  // namespace

// The tail starts at chunk nck-2 of the last segment (its first chunk when it has fewer).
cudaError_t launch_state_tail(const PrefillPlan &p, int tail_chunks, cudaStream_t s) {
  if (!p.h_final || p.L == 0) return cudaSuccess;
  const int t_b = (p.n_seg - 1) * p.seg_len;
  const int nck = (p.L - t_b + 127) / 128;
  const int t_tail = t_b + 128 * (nck > tail_chunks ? nck - tail_chunks : 0);
  state_tail_kernel<<<dim3(p.H, p.B), kTailThreads, 0, s>>>(
      (const __nv_bfloat16 *)p.xBC, p.xs, (const __nv_bfloat16 *)p.conv_w, (const __nv_bfloat16 *)p.conv_b,
      (const __nv_bfloat16 *)p.csi, p.dte_hm, p.cs_hm, p.h_final, p.L, p.H, p.hpg, p.conv_dim, p.d_inner, p.W,
      p.Lpad, t_tail);
  return cudaGetLastError();
}

}  // namespace ssd
