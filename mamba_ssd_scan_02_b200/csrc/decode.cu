// decode.cu -- one decode step of the Mamba-2 mixer scan (one new token per batch row).
//
// Per batch row b and head h (group g = h / (H/G)):
//   cache' = cache[1:] ++ xBC_t            (the conv cache holds the last W raw inputs)
//   u      = silu(conv_b + sum_k conv_w[:,k] * cache'[k])
//   dt     = clamp(softplus(dt_raw + dt_bias_h));  a = exp(dt A_h)
//   h      = a h + dt x B^T                 (P x N, fp32, in place)
//   y      = h C + D_h x;  then the z-gated RMSNorm over each norm group
// The fp32 state follows the float32 SSM-cache requirement (neurohive.io article on
// Nemotron Nano 2, section "Deployment and usage").
//
// The step is bound by HBM: it reads and writes the whole fp32 state once (32 KiB per head).
// One CTA covers one (batch row, group): it computes the conv for the group's x, B and C
// channels once, then its warps stream the heads' states with 16-byte loads (8 rows of a head
// in flight per warp, streaming cache hints), and finally applies the gated norm to the
// group's channels, which is local because norm groups nest inside SSM groups.
#include "common.cuh"
#include "plan.h"

namespace ssd {
namespace {

constexpr int kDecThreads = 512;
constexpr int kRowsInFlight = 8;

template <typename T, int W>
__global__ void __launch_bounds__(kDecThreads) decode_kernel(DecodePlan p) {
  extern __shared__ __align__(16) float dsm[];
  const int g = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int nx = p.hpg * kHeadDim;          // x channels of the group
  float *ux = dsm;                          // [nx]
  float *uB = ux + nx;                      // [N]
  float *uC = uB + kDState;                 // [N]
  float *ys = uC + kDState;                 // [nx]
  float *dts = ys + nx;                     // [hpg]
  __shared__ float red[32];

  // ---- conv of the group's channels (x: nx, B: N, C: N), cache shift -------------------
  const int nvec = (nx + 2 * kDState) / 8;
  const T *xrow = reinterpret_cast<const T *>(p.xBC) + (long long)b * p.xs;
  for (int v = tid; v < nvec; v += kDecThreads) {
    int ch, local;
    float *dst;
    if (v * 8 < nx) {
      local = v * 8; ch = g * nx + local; dst = ux + local;
    } else if (v * 8 < nx + kDState) {
      local = v * 8 - nx; ch = p.d_inner + g * kDState + local; dst = uB + local;
    } else {
      local = v * 8 - nx - kDState; ch = p.d_inner + p.G * kDState + g * kDState + local; dst = uC + local;
    }
    float cur[8];
    load8(xrow + ch, cur);
    if (W == 0) {
#pragma unroll
      for (int i = 0; i < 8; ++i) dst[i] = cur[i];
      continue;
    }
    const long long cbase = (long long)b * W * p.conv_dim + ch;
    const T *csi = reinterpret_cast<const T *>(p.csi);
    T *cso = reinterpret_cast<T *>(p.cso);
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      acc[i] = p.conv_b ? io<T>::ld(reinterpret_cast<const T *>(p.conv_b) + ch + i) : 0.f;
      acc[i] += io<T>::ld(reinterpret_cast<const T *>(p.conv_w) + (long long)(ch + i) * W + (W - 1)) * cur[i];
    }
#pragma unroll
    for (int k = 0; k + 1 < W; ++k) {
      // new cache row k = old row k+1 (raw 16-byte copy, bit-exact)
      const T *src = csi + cbase + (long long)(k + 1) * p.conv_dim;
      if (sizeof(T) == 2) {
        *reinterpret_cast<uint4 *>(cso + cbase + (long long)k * p.conv_dim) = *reinterpret_cast<const uint4 *>(src);
      } else {
        *reinterpret_cast<uint4 *>(cso + cbase + (long long)k * p.conv_dim) = *reinterpret_cast<const uint4 *>(src);
        *reinterpret_cast<uint4 *>(cso + cbase + (long long)k * p.conv_dim + 4) = *reinterpret_cast<const uint4 *>(src + 4);
      }
      float hv[8];
      load8(src, hv);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        acc[i] += io<T>::ld(reinterpret_cast<const T *>(p.conv_w) + (long long)(ch + i) * W + k) * hv[i];
    }
    {  // newest cache row = the raw new input
      T *dstc = cso + cbase + (long long)(W - 1) * p.conv_dim;
      if (sizeof(T) == 2) {
        *reinterpret_cast<uint4 *>(dstc) = *reinterpret_cast<const uint4 *>(xrow + ch);
      } else {
        *reinterpret_cast<uint4 *>(dstc) = *reinterpret_cast<const uint4 *>(xrow + ch);
        *reinterpret_cast<uint4 *>(dstc + 4) = *reinterpret_cast<const uint4 *>(xrow + ch + 4);
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) dst[i] = silu(acc[i]);
  }
  if (tid < p.hpg) {
    const int h = g * p.hpg + tid;
    dts[tid] = effective_dt(io<T>::ld(reinterpret_cast<const T *>(p.dt) + (long long)b * p.ds + h),
                            p.dt_bias[h], p.softplus, p.dt_min, p.dt_max);
  }
  __syncthreads();

  // ---- state update and read-out: warp w streams heads w, w+16, ... --------------------
  const float4 B4 = reinterpret_cast<const float4 *>(uB)[lane];
  const float4 C4 = reinterpret_cast<const float4 *>(uC)[lane];
  for (int hi = warp; hi < p.hpg; hi += kDecThreads / 32) {
    const int h = g * p.hpg + hi;
    const float dt = dts[hi];
    const float a = __expf(dt * p.A[h]);
    const float Dh = p.D[h];
    float4 *st = reinterpret_cast<float4 *>(p.state + ((long long)b * p.H + h) * kHeadDim * kDState);
    for (int p0 = 0; p0 < kHeadDim; p0 += kRowsInFlight) {
      float4 hv[kRowsInFlight];
#pragma unroll
      for (int i = 0; i < kRowsInFlight; ++i) hv[i] = __ldcs(st + (p0 + i) * (kDState / 4) + lane);
#pragma unroll
      for (int i = 0; i < kRowsInFlight; ++i) {
        const float xp = ux[hi * kHeadDim + p0 + i];
        const float dx = dt * xp;
        float4 v = hv[i];
        v.x = a * v.x + dx * B4.x;
        v.y = a * v.y + dx * B4.y;
        v.z = a * v.z + dx * B4.z;
        v.w = a * v.w + dx * B4.w;
        __stcs(st + (p0 + i) * (kDState / 4) + lane, v);
        float part = v.x * C4.x + v.y * C4.y + v.z * C4.z + v.w * C4.w;
        part = warp_sum(part);
        if (lane == 0) ys[hi * kHeadDim + p0 + i] = part + Dh * xp;
      }
    }
  }
  __syncthreads();

  // ---- gated RMSNorm (norm groups nest in the SSM group) and output ----------------------
  T *yout = reinterpret_cast<T *>(p.y) + (long long)b * p.ys + g * nx;
  if (p.norm_groups == 0) {
    for (int i = tid; i < nx; i += kDecThreads) io<T>::st(yout + i, ys[i]);
    return;
  }
  const T *zr = reinterpret_cast<const T *>(p.z) + (long long)b * p.zs + g * nx;
  const int sub = p.norm_groups / p.G;  // norm groups inside this SSM group
  const int gs = nx / sub;
  if (!p.nbg) {  // gate first (the default); else normalise y first and gate below
    for (int i = tid; i < nx; i += kDecThreads) ys[i] *= silu(io<T>::ld(zr + i));
    __syncthreads();
  }
  for (int k = 0; k < sub; ++k) {
    float ss = 0.f;
    for (int i = tid; i < gs; i += kDecThreads) ss += ys[k * gs + i] * ys[k * gs + i];
    ss = warp_sum(ss);
    if (lane == 0) red[warp] = ss;
    __syncthreads();
    if (warp == 0) {
      float t = lane < kDecThreads / 32 ? red[lane] : 0.f;
      t = warp_sum(t);
      if (lane == 0) red[0] = t;
    }
    __syncthreads();
    const float r = rsqrtf(red[0] / gs + p.eps);
    __syncthreads();
    const T *wr = reinterpret_cast<const T *>(p.norm_w);
    for (int i = tid; i < gs; i += kDecThreads) {
      const int c = k * gs + i;
      const float gate = p.nbg ? silu(io<T>::ld(zr + c)) : 1.f;
      io<T>::st(yout + c, ys[c] * r * (wr ? io<T>::ld(wr + g * nx + c) : 1.f) * gate);
    }
  }
}

template <typename T, int W>
cudaError_t launch_w(const DecodePlan &p, cudaStream_t s) {
  const size_t smem = sizeof(float) * (2 * p.hpg * kHeadDim + 2 * kDState + p.hpg + 4);
  cudaError_t e = set_smem_attr(decode_kernel<T, W>, smem, s);
  if (e != cudaSuccess) return e;
  decode_kernel<T, W><<<dim3(p.G, p.B), kDecThreads, smem, s>>>(p);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_t(const DecodePlan &p, cudaStream_t s) {
  switch (p.W) {
    case 0: return launch_w<T, 0>(p, s);
    case 1: return launch_w<T, 1>(p, s);
    case 2: return launch_w<T, 2>(p, s);
    case 3: return launch_w<T, 3>(p, s);
    default: return launch_w<T, 4>(p, s);
  }
}

}  // namespace

cudaError_t launch_decode(const DecodePlan &p, cudaStream_t s) {
  return p.bf16 ? launch_t<__nv_bfloat16>(p, s) : launch_t<float>(p, s);
}

}  // namespace ssd
