// common.cuh -- small device helpers shared by the libssd kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ssd.h"

namespace ssd {

constexpr int kHeadDim = 64;   // P
constexpr int kDState = 128;   // N

// Kernels that can fail (a bounded wait that gives up, a checked index) receive a pointer to
// the library's device error word and latch the first failure there instead of trapping;
// ssd_get_device_error() reads and clears it.
__device__ __forceinline__ void latch_error(int *err, int code) {
  if (err) atomicCAS(err, 0, code);
}

// ---- index checks of the debug build ---------------------------------------------------------
// Built with -DSSD_DEBUG_BOUNDS (libssd_debug.so), the kernels check the index of each global
// store against the extent of the buffer it writes: an index outside [0, extent) latches
// SSD_ERR_DEVICE_BOUNDS in the device error word and the store is skipped (no trap).  In the
// normal build the check is the constant true and costs nothing.
#ifdef SSD_DEBUG_BOUNDS
__device__ __forceinline__ bool in_bounds(long long i, long long extent, int *err) {
  if (i >= 0 && i < extent) return true;
  latch_error(err, (int)SSD_ERR_DEVICE_BOUNDS);
  return false;
}
#else
__device__ __forceinline__ constexpr bool in_bounds(long long, long long, int *) { return true; }
#endif

// ---- row geometry of a batch -----------------------------------------------------------------
// A uniform batch stores batch row b's token t at row b*L + t.  A variable-length batch packs
// its sequences back to back: sequence b is rows cu[b] .. cu[b+1]-1 (cu: device offsets, B + 1
// of them) and L is the longest length, which sizes the grids.
__device__ __forceinline__ long long seq_base(const int *cu, int b, int L) {
  return cu ? (long long)cu[b] : (long long)b * L;
}
__device__ __forceinline__ int seq_len(const int *cu, int b, int L) { return cu ? cu[b + 1] - cu[b] : L; }

// ---- element loads / stores in the io dtype ------------------------------------------------
template <typename T> struct io;
template <> struct io<float> {
  static __device__ __forceinline__ float ld(const float *p) { return *p; }
  static __device__ __forceinline__ void st(float *p, float v) { *p = v; }
};
template <> struct io<__nv_bfloat16> {
  static __device__ __forceinline__ float ld(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
  static __device__ __forceinline__ void st(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }
};

// 8 consecutive elements as floats (one 16-byte load for bf16, two for fp32).
__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float (&v)[8]) {
  uint4 u = *reinterpret_cast<const uint4 *>(p);
  const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void load8(const float *p, float (&v)[8]) {
  float4 a = *reinterpret_cast<const float4 *>(p);
  float4 b = *reinterpret_cast<const float4 *>(p + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void store8(__nv_bfloat16 *p, const float (&v)[8]) {
  uint4 u;
  __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
  *reinterpret_cast<uint4 *>(p) = u;
}
__device__ __forceinline__ void store8(__half *p, const float (&v)[8]) {
  uint4 u;
  __half2 *h = reinterpret_cast<__half2 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2half2_rn(v[2 * i], v[2 * i + 1]);
  *reinterpret_cast<uint4 *>(p) = u;
}
__device__ __forceinline__ void store8(float *p, const float (&v)[8]) {
  *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
  *reinterpret_cast<float4 *>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
}

// ---- activations ---------------------------------------------------------------------------
// x * sigmoid(x) with the hardware exponential and the fast reciprocal-based division (a few
// ulp of fp32; for x < -87 the denominator overflows and the result is 0, as in fp32 exactly).
__device__ __forceinline__ float silu(float x) { return __fdividef(x, 1.0f + __expf(-x)); }

// softplus(x) = log(1 + e^x); above 20 it equals x to fp32 precision.
__device__ __forceinline__ float softplus(float x) { return x > 20.0f ? x : log1pf(__expf(x)); }

__device__ __forceinline__ float effective_dt(float raw, float bias, int use_softplus, float lo,
                                              float hi) {
  float v = raw + bias;
  if (use_softplus) v = softplus(v);
  return fminf(fmaxf(v, lo), hi);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Opt a kernel into more than 48 KiB of dynamic shared memory.  The attribute persists, so
// while a stream is being captured into a graph (where it was set by an earlier launch) the
// call is skipped.
template <typename Kernel>
inline cudaError_t set_smem_attr(Kernel kernel, size_t bytes, cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) == cudaSuccess && cs != cudaStreamCaptureStatusNone)
    return cudaSuccess;
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

}  // namespace ssd
