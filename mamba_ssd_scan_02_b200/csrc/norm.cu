// norm.cu -- the z-gated RMSNorm applied to the scan output, and the plain RMSNorm at the
// mixer input (as a per-row factor and a folded weight, applied by the in_proj GEMM).  The Nemotron Nano 2 layers normalise with RMSNorm ("NVIDIA Nemotron Nano 2"
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

// y as the scan left it: fp32 (the CUDA-core path) or fp16 (the tensor-core path).
__device__ __forceinline__ float ld_y(const float *p) { return *p; }
__device__ __forceinline__ float ld_y(const __half *p) { return __half2float(*p); }

// One CTA per (row, norm group).  y is [rows, d_inner] dense (YT: float or __half); z/out/w in
// the io dtype.
template <typename T, typename YT>
__global__ void __launch_bounds__(kNormThreads) gated_norm_kernel(
    const YT *__restrict__ y, const T *__restrict__ z, long long zs, const T *__restrict__ w,
    T *__restrict__ out, long long os, int d_inner, int gs, float eps, int nbg, long long out_extent, int *err) {
  __shared__ float red[32];
  const long long row = blockIdx.x;
  const int c0 = blockIdx.y * gs;
  const YT *yr = y + row * d_inner + c0;
  const T *zr = z + row * zs + c0;
  float ss = 0.f;
  for (int i = threadIdx.x; i < gs; i += kNormThreads) {
    const float yv = ld_y(yr + i);
    const float gv = nbg ? yv : yv * silu(io<T>::ld(zr + i));
    ss += gv * gv;
  }
  ss = block_sum(ss, red);
  const float r = rsqrtf(ss / gs + eps);
  T *orow = out + row * os + c0;
  for (int i = threadIdx.x; i < gs; i += kNormThreads) {
    const float sz = silu(io<T>::ld(zr + i));
    const float yv = ld_y(yr + i);
    const float gv = nbg ? yv : yv * sz;
    if (in_bounds(row * os + c0 + i, out_extent, err))
      io<T>::st(orow + i, gv * r * (w ? io<T>::ld(w + c0 + i) : 1.f) * (nbg ? sz : 1.f));
  }
}

// The RMSNorm's per-row factor alone (the projection that follows applies it): one CTA per row.
__global__ void __launch_bounds__(kNormThreads) rms_rowscale_bf16_kernel(
    const __nv_bfloat16 *__restrict__ x, float *__restrict__ r, int width, float eps) {
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
  if (threadIdx.x == 0) r[row] = rsqrtf(ss / width + eps);
}

// W'[n][k] = W[n][k] * w[k], 8 elements per thread (16-byte accesses).
__global__ void fold_cols_bf16_kernel(const __nv_bfloat16 *__restrict__ W, const __nv_bfloat16 *__restrict__ w,
                                      __nv_bfloat16 *__restrict__ out, long long n8, int K) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n8; i += (long long)gridDim.x * blockDim.x) {
    const int k = (int)((i * 8) % K);
    float v[8], wv[8];
    load8(W + i * 8, v);
    load8(w + k, wv);
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] *= wv[j];
    store8(out + i * 8, v);
  }
}

}  // namespace

// 8 consecutive channels of y (streaming loads: each is read once)
__device__ __forceinline__ void ld_y8(const float *p, float (&v)[8]) {
  const float4 a = __ldcs(reinterpret_cast<const float4 *>(p)), b = __ldcs(reinterpret_cast<const float4 *>(p + 4));
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void ld_y8(const __half *p, float (&v)[8]) {
  const uint4 u = __ldcs(reinterpret_cast<const uint4 *>(p));
  const __half2 *h = reinterpret_cast<const __half2 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __half22float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}

// The same for bf16 tensors in one pass: a CTA of gs / 8 threads per (row, norm group), each
// thread holding 8 consecutive channels in registers (16-byte loads and stores).
template <typename YT>
__global__ void __launch_bounds__(1024) gated_norm_v8_kernel(
    const YT *__restrict__ y, const __nv_bfloat16 *__restrict__ z, long long zs,
    const __nv_bfloat16 *__restrict__ w, __nv_bfloat16 *__restrict__ out, long long os, int d_inner,
    int gs, float eps, int nbg, long long out_extent, int *err) {
  __shared__ float red[32];
  const long long row = blockIdx.x;
  const int c = blockIdx.y * gs + 8 * threadIdx.x;
  float yv[8], zv[8], g[8];
  ld_y8(y + row * d_inner + c, yv);
  load8(z + row * zs + c, zv);
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
  if (in_bounds(row * os + c + 7, out_extent, err)) store8(out + row * os + c, g);
}

cudaError_t launch_gated_norm(const PrefillPlan &p, cudaStream_t s) {
  const int gs = p.d_inner / p.norm_groups;
  dim3 grid((unsigned)p.rows, p.norm_groups);
  const bool v8 = p.bf16 && gs % 256 == 0 && gs / 8 <= 1024 &&  // whole warps of 8 channels
                  (reinterpret_cast<uintptr_t>(p.norm_w) & 15u) == 0;
  const auto *z = (const __nv_bfloat16 *)p.z;
  const auto *w = (const __nv_bfloat16 *)p.norm_w;
  auto *o = (__nv_bfloat16 *)p.y;
  const long long ext = checked_extent(p, (p.rows - 1) * p.ys + p.d_inner);
  if (p.yh) {  // tensor path: fp16 y, bf16 tensors
    if (!p.bf16) return cudaErrorInvalidValue;
    if (v8)
      gated_norm_v8_kernel<__half><<<grid, gs / 8, 0, s>>>(p.yh, z, p.zs, w, o, p.ys, p.d_inner, gs, p.eps, p.nbg,
                                                          ext, p.err);
    else
      gated_norm_kernel<__nv_bfloat16, __half><<<grid, kNormThreads, 0, s>>>(p.yh, z, p.zs, w, o, p.ys,
                                                                             p.d_inner, gs, p.eps, p.nbg, ext, p.err);
  } else if (v8) {
    gated_norm_v8_kernel<float><<<grid, gs / 8, 0, s>>>(p.yf, z, p.zs, w, o, p.ys, p.d_inner, gs, p.eps, p.nbg, ext,
                                                        p.err);
  } else if (p.bf16) {
    gated_norm_kernel<__nv_bfloat16, float><<<grid, kNormThreads, 0, s>>>(p.yf, z, p.zs, w, o, p.ys, p.d_inner,
                                                                          gs, p.eps, p.nbg, ext, p.err);
  } else {
    gated_norm_kernel<float, float><<<grid, kNormThreads, 0, s>>>(p.yf, (const float *)p.z, p.zs,
                                                                  (const float *)p.norm_w, (float *)p.y,
                                                                  p.ys, p.d_inner, gs, p.eps, p.nbg, ext, p.err);
  }
  return cudaGetLastError();
}


cudaError_t launch_rms_rowscale_bf16(const void *x, float *r, long long rows, int width, float eps,
                                     cudaStream_t s) {
  if (width % 8) return cudaErrorInvalidValue;
  rms_rowscale_bf16_kernel<<<(unsigned)rows, kNormThreads, 0, s>>>((const __nv_bfloat16 *)x, r, width, eps);
  return cudaGetLastError();
}

cudaError_t launch_fold_cols_bf16(const void *W, const void *w, void *out, long long rows, int K,
                                  cudaStream_t s) {
  if (K % 8) return cudaErrorInvalidValue;
  const long long n8 = rows * K / 8;
  long long blocks = (n8 + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  fold_cols_bf16_kernel<<<(unsigned)blocks, 256, 0, s>>>((const __nv_bfloat16 *)W, (const __nv_bfloat16 *)w,
                                                         (__nv_bfloat16 *)out, n8, K);
  return cudaGetLastError();
}

}  // namespace ssd
