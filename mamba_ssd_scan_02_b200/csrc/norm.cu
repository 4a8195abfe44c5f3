// norm.cu -- the z-gated RMSNorm applied to the scan output, and the plain RMSNorm at the
// mixer input.  The Nemotron Nano 2 layers normalise with RMSNorm ("NVIDIA Nemotron Nano 2"
// summary, section "Method"); in the Mamba-2 mixer the scan output is gated by SiLU(z) and
// then normalised over groups of d_inner / norm_groups consecutive channels:
//   g = y * silu(z);   out = g / sqrt(mean_group(g^2) + eps) * w
// or, normalising before the gate (the norm_before_gate variant):
//   out = y / sqrt(mean_group(y^2) + eps) * w * silu(z)
#include <stdint.h>

#include "common.cuh"
#include "plan.h"

namespace ssd {
namespace {

constexpr int kNormThreads = 256;

__device__ float block_sum(float v, float *red) {
  v = warp_sum(v);
  const int w = threadIdx.x / 32, l = threadIdx.x % 32;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float t = threadIdx.x < blockDim.x / 32 ? red[threadIdx.x] : 0.f;
  if (w == 0) {
    t = warp_sum(t);
    if (l == 0) red[0] = t;
  }
  __syncthreads();
  return red[0];
}

// One CTA per (row, norm group).  y is fp32 [rows, d_inner] dense; z/out/w in the io dtype.
template <typename T>
__global__ void __launch_bounds__(kNormThreads) gated_norm_kernel(
    const float *__restrict__ y, const T *__restrict__ z, long long zs, const T *__restrict__ w,
    T *__restrict__ out, long long os, int d_inner, int gs, float eps, int L, int nbg) {
  __shared__ float red[32];
  const long long row = blockIdx.x;
  const int c0 = blockIdx.y * gs;
  const float *yr = y + row * d_inner + c0;
  const T *zr = z + row * zs + c0;
  float ss = 0.f;
  for (int i = threadIdx.x; i < gs; i += kNormThreads) {
    const float gv = nbg ? yr[i] : yr[i] * silu(io<T>::ld(zr + i));
    ss += gv * gv;
  }
  ss = block_sum(ss, red);
  const float r = rsqrtf(ss / gs + eps);
  T *orow = out + row * os + c0;
  for (int i = threadIdx.x; i < gs; i += kNormThreads) {
    const float sz = silu(io<T>::ld(zr + i));
    const float gv = nbg ? yr[i] : yr[i] * sz;
    io<T>::st(orow + i, gv * r * (w ? io<T>::ld(w + c0 + i) : 1.f) * (nbg ? sz : 1.f));
  }
}

__global__ void __launch_bounds__(kNormThreads) rmsnorm_bf16_kernel(
    const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ w,
    __nv_bfloat16 *__restrict__ out, int width, float eps) {
  __shared__ float red[32];
  const long long row = blockIdx.x;
  const __nv_bfloat16 *xr = x + row * width;
  float ss = 0.f;
  for (int i = threadIdx.x * 8; i < width; i += kNormThreads * 8) {
    float v[8];
    load8(xr + i, v);
#pragma unroll
    for (int k = 0; k < 8; ++k) ss += v[k] * v[k];
  }
  ss = block_sum(ss, red);
  const float r = rsqrtf(ss / width + eps);
  for (int i = threadIdx.x * 8; i < width; i += kNormThreads * 8) {
    float v[8], wv[8];
    load8(xr + i, v);
    if (w) load8(w + i, wv);
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = v[k] * r * (w ? wv[k] : 1.f);
    store8(out + row * width + i, v);
  }
}

}  // namespace

// The same for bf16 tensors in one pass: a CTA of gs / 8 threads per (row, norm group), each
// thread holding 8 consecutive channels in registers (16-byte loads and stores).
__global__ void __launch_bounds__(1024) gated_norm_v8_kernel(
    const float *__restrict__ y, const __nv_bfloat16 *__restrict__ z, long long zs,
    const __nv_bfloat16 *__restrict__ w, __nv_bfloat16 *__restrict__ out, long long os, int d_inner,
    int gs, float eps, int nbg) {
  __shared__ float red[32];
  const long long row = blockIdx.x;
  const int c = blockIdx.y * gs + 8 * threadIdx.x;
  const float4 ya = __ldcs(reinterpret_cast<const float4 *>(y + row * d_inner + c));
  const float4 yb = __ldcs(reinterpret_cast<const float4 *>(y + row * d_inner + c + 4));
  float zv[8], g[8];
  load8(z + row * zs + c, zv);
  const float yv[8] = {ya.x, ya.y, ya.z, ya.w, yb.x, yb.y, yb.z, yb.w};
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    zv[i] = silu(zv[i]);
    g[i] = nbg ? yv[i] : yv[i] * zv[i];
    ss = fmaf(g[i], g[i], ss);
  }
  ss = block_sum(ss, red);
  const float r = rsqrtf(ss / gs + eps);
  float wv[8];
  if (w) {
    load8(w + c, wv);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) wv[i] = 1.f;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) g[i] *= r * wv[i] * (nbg ? zv[i] : 1.f);
  store8(out + row * os + c, g);
}

// Second half of the gated norm fused into the tensor-core scan.  The scan's output stage
// has gated each token's head (g = y * silu(z), or g = y when normalising first) and stored
//   q_h   = g / s_h  in fp16, with s_h = sqrt(mean of g^2 over the head's 64 channels)
//   ssq_h = sum of g^2 over those channels (fp32, per token row and head),
// so |q| <= 8 and fp16 keeps 11 significant bits of it with no risk of overflow.  A norm group
// covers whole heads, and its statistic is the sum of its heads' ssq:
//   out = q * s_h * rsqrt(sum_{h in group} ssq_h / gs + eps) * w   (* silu(z) normalising first).
// One CTA per token row: the row's per-head factors are formed in shared memory, then every
// thread rescales 8 channels at a time (16-byte loads and stores).
constexpr int kRescaleThreads = 256;

__global__ void __launch_bounds__(kRescaleThreads) norm_rescale_kernel(
    const __half *__restrict__ q, const float *__restrict__ ssq, const __nv_bfloat16 *__restrict__ z,
    long long zs, const __nv_bfloat16 *__restrict__ w, __nv_bfloat16 *__restrict__ out, long long os,
    int H, int hpn, int ng, int d_inner, float eps, int nbg) {
  extern __shared__ float rsm[];
  float *sq = rsm, *fac = rsm + H, *gsum = rsm + 2 * H;
  const long long row = blockIdx.x;
  for (int i = threadIdx.x; i < H; i += kRescaleThreads) sq[i] = ssq[row * H + i];
  __syncthreads();
  for (int gi = threadIdx.x; gi < ng; gi += kRescaleThreads) {  // fixed order: reproducible
    float t = 0.f;
    for (int j = 0; j < hpn; ++j) t += sq[gi * hpn + j];
    gsum[gi] = rsqrtf(t / (float)(hpn * kHeadDim) + eps);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < H; i += kRescaleThreads)
    fac[i] = sqrtf(sq[i] * (1.f / kHeadDim)) * gsum[i / hpn];
  __syncthreads();
  const __half *qr = q + row * d_inner;
  for (int c = threadIdx.x * 8; c < d_inner; c += kRescaleThreads * 8) {
    const uint4 qu = __ldcs(reinterpret_cast<const uint4 *>(qr + c));
    const __half2 *q2 = reinterpret_cast<const __half2 *>(&qu);
    const float f = fac[c / kHeadDim];
    float v[8], wv[8];
    if (w) {
      load8(w + c, wv);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) wv[i] = 1.f;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 qf = __half22float2(q2[i]);
      v[2 * i] = qf.x * f * wv[2 * i];
      v[2 * i + 1] = qf.y * f * wv[2 * i + 1];
    }
    if (nbg) {
      float zv[8];
      load8(z + row * zs + c, zv);
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] *= silu(zv[i]);
    }
    store8(out + row * os + c, v);
  }
}

cudaError_t launch_norm_rescale(const PrefillPlan &p, cudaStream_t s) {
  const int hpn = p.H / p.norm_groups;
  const size_t smem = (size_t)(2 * p.H + p.norm_groups) * sizeof(float);
  if (smem > 48 * 1024) return cudaErrorInvalidValue;
  norm_rescale_kernel<<<(unsigned)p.rows, kRescaleThreads, smem, s>>>(
      p.qn, p.ssq, (const __nv_bfloat16 *)p.z, p.zs, (const __nv_bfloat16 *)p.norm_w,
      (__nv_bfloat16 *)p.y, p.ys, p.H, hpn, p.norm_groups, p.d_inner, p.eps, p.nbg);
  return cudaGetLastError();
}

cudaError_t launch_gated_norm(const PrefillPlan &p, cudaStream_t s) {
  const int gs = p.d_inner / p.norm_groups;
  dim3 grid((unsigned)p.rows, p.norm_groups);
  const bool v8 = p.bf16 && gs % 256 == 0 && gs / 8 <= 1024 &&  // whole warps of 8 channels
                  (reinterpret_cast<uintptr_t>(p.norm_w) & 15u) == 0;
  if (v8)
    gated_norm_v8_kernel<<<grid, gs / 8, 0, s>>>(p.yf, (const __nv_bfloat16 *)p.z, p.zs,
                                                 (const __nv_bfloat16 *)p.norm_w, (__nv_bfloat16 *)p.y,
                                                 p.ys, p.d_inner, gs, p.eps, p.nbg);
  else if (p.bf16)
    gated_norm_kernel<__nv_bfloat16><<<grid, kNormThreads, 0, s>>>(
        p.yf, (const __nv_bfloat16 *)p.z, p.zs, (const __nv_bfloat16 *)p.norm_w,
        (__nv_bfloat16 *)p.y, p.ys, p.d_inner, gs, p.eps, p.L, p.nbg);
  else
    gated_norm_kernel<float><<<grid, kNormThreads, 0, s>>>(p.yf, (const float *)p.z, p.zs,
                                                           (const float *)p.norm_w, (float *)p.y,
                                                           p.ys, p.d_inner, gs, p.eps, p.L, p.nbg);
  return cudaGetLastError();
}


cudaError_t launch_rmsnorm_bf16(const void *x, const void *w, void *out, long long rows, int width,
                                float eps, cudaStream_t s) {
  rmsnorm_bf16_kernel<<<(unsigned)rows, kNormThreads, 0, s>>>(
      (const __nv_bfloat16 *)x, (const __nv_bfloat16 *)w, (__nv_bfloat16 *)out, width, eps);
  return cudaGetLastError();
}

}  // namespace ssd
