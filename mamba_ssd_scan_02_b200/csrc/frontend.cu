// frontend.cu -- the scan's front end: causal depthwise conv1d (window W <= 4) + SiLU over
// the raw x|B|C channels, the effective time step softplus(dt_raw + dt_bias) with clamp, and
// the conv cache carried to the next call (the last W raw inputs, copied bit for bit).
//
// The conv of token t for channel c is silu(conv_b[c] + sum_k conv_w[c,k] * x[t-(W-1)+k, c]);
// inputs before the first token come from the incoming cache (row W-1 = the newest).  This is
// the Mamba-2 short convolution of window 4 in the Nemotron Nano 2 layers ("NVIDIA Nemotron
// Nano 2" summary, section "Method").
#include "common.cuh"
#include "plan.h"

namespace ssd {
namespace {

constexpr int kConvTokens = 32;  // tokens per thread (sliding window kept in registers)

// One thread: 8 consecutive channels x kConvTokens consecutive tokens of one batch row.
// 16-byte vector loads along the channel dimension are coalesced across the warp.
template <typename T, int W>
__global__ void __launch_bounds__(128) conv_silu_kernel(const T *__restrict__ xBC, long long xs,
                                                        const T *__restrict__ csi,
                                                        const T *__restrict__ w,
                                                        const T *__restrict__ bias,
                                                        float *__restrict__ u, int L, int C) {
  const int c8 = (blockIdx.x * blockDim.x + threadIdx.x) * 8;
  if (c8 >= C) return;
  const int b = blockIdx.z;
  const int t0 = blockIdx.y * kConvTokens;
  const T *xrow = xBC + (long long)b * L * xs;
  float wt[4][8], bs[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    bs[i] = bias ? io<T>::ld(bias + c8 + i) : 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) wt[k][i] = (k < W) ? io<T>::ld(w + (long long)(c8 + i) * W + k) : 0.f;
  }
  // hist[j] holds time t-3+j (j = 0..2) before processing token t
  float hist[3][8];
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    const int tau = t0 - 3 + j;
    if (W > 0 && tau >= 0) {
      load8(xrow + (long long)tau * xs + c8, hist[j]);
    } else if (csi && W > 0 && W + tau >= 0) {
      load8(csi + ((long long)b * W + (W + tau)) * C + c8, hist[j]);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) hist[j][i] = 0.f;
    }
  }
  const int t1 = min(L, t0 + kConvTokens);
  for (int t = t0; t < t1; ++t) {
    float cur[8], out[8];
    load8(xrow + (long long)t * xs + c8, cur);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (W == 0) {
        out[i] = cur[i];
        continue;
      }
      // tap k multiplies time t-(W-1)+k: k = W-1 is cur, k = W-1-j is hist[3-j]
      float acc = bs[i] + wt[W > 0 ? W - 1 : 0][i] * cur[i];
#pragma unroll
      for (int j = 1; j < W; ++j) acc += wt[W - 1 - j][i] * hist[3 - j][i];
      out[i] = silu(acc);
    }
    store8(u + ((long long)b * L + t) * C + c8, out);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      hist[0][i] = hist[1][i];
      hist[1][i] = hist[2][i];
      hist[2][i] = cur[i];
    }
  }
}

template <typename T>
__global__ void dt_kernel(const T *__restrict__ dt, long long ds, const float *__restrict__ bias,
                          float *__restrict__ dte, long long rows, int H, int sp, float lo, float hi) {
  const long long n = rows * H;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const long long r = i / H;
    const int h = (int)(i % H);
    dte[i] = effective_dt(io<T>::ld(dt + r * ds + h), bias[h], sp, lo, hi);
  }
}

// conv_state_out[b, k, :] = raw input of time L-W+k (from the incoming cache when negative).
// Copies 16-byte words without conversion, so the carried cache is bit-exact.
template <int ELT>
__global__ void conv_state_out_kernel(const char *__restrict__ xBC, long long xs_bytes,
                                      const char *__restrict__ csi, char *__restrict__ cso, int B,
                                      int L, int W, int C) {
  const long long row_bytes = (long long)C * ELT;
  const long long vec_per_row = row_bytes / 16;
  const long long n = (long long)B * W * vec_per_row;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const long long v = i % vec_per_row;
    const int k = (int)((i / vec_per_row) % W);
    const int b = (int)(i / (vec_per_row * W));
    const int tau = L - W + k;
    uint4 val = make_uint4(0, 0, 0, 0);
    if (tau >= 0)
      val = *reinterpret_cast<const uint4 *>(xBC + ((long long)b * L + tau) * xs_bytes + v * 16);
    else if (csi)
      val = *reinterpret_cast<const uint4 *>(csi + ((long long)b * W + (W + tau)) * row_bytes + v * 16);
    *reinterpret_cast<uint4 *>(cso + ((long long)b * W + k) * row_bytes + v * 16) = val;
  }
}

// seqlen == 0: the state passes through unchanged and so does the conv cache.
__global__ void carry_state_kernel(const float *__restrict__ h0, float *__restrict__ hf, long long n) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x)
    hf[i] = h0 ? h0[i] : 0.f;
}

int grid_for(long long n, int threads) {
  long long g = (n + threads - 1) / threads;
  return (int)(g < 1 ? 1 : (g > 148 * 16 ? 148 * 16 : g));
}

}  // namespace

template <typename T, int W>
static void conv_launch(const PrefillPlan &p, dim3 grid, int threads, cudaStream_t s) {
  conv_silu_kernel<T, W><<<grid, threads, 0, s>>>((const T *)p.xBC, p.xs, (const T *)p.csi,
                                                   (const T *)p.conv_w, (const T *)p.conv_b, p.u,
                                                   p.L, p.conv_dim);
}

template <typename T>
static void conv_dispatch(const PrefillPlan &p, dim3 grid, int threads, cudaStream_t s) {
  switch (p.W) {
    case 0: conv_launch<T, 0>(p, grid, threads, s); break;
    case 1: conv_launch<T, 1>(p, grid, threads, s); break;
    case 2: conv_launch<T, 2>(p, grid, threads, s); break;
    case 3: conv_launch<T, 3>(p, grid, threads, s); break;
    default: conv_launch<T, 4>(p, grid, threads, s); break;
  }
}

cudaError_t launch_conv_silu_f32(const PrefillPlan &p, cudaStream_t s) {
  const int threads = 128;
  dim3 grid((p.conv_dim / 8 + threads - 1) / threads, (p.L + kConvTokens - 1) / kConvTokens, p.B);
  if (p.bf16)
    conv_dispatch<__nv_bfloat16>(p, grid, threads, s);
  else
    conv_dispatch<float>(p, grid, threads, s);
  return cudaGetLastError();
}

cudaError_t launch_dt(const PrefillPlan &p, cudaStream_t s) {
  const long long rows = (long long)p.B * p.L;
  const int g = grid_for(rows * p.H, 256);
  if (p.bf16)
    dt_kernel<__nv_bfloat16><<<g, 256, 0, s>>>((const __nv_bfloat16 *)p.dt, p.ds, p.dt_bias, p.dte,
                                                rows, p.H, p.softplus, p.dt_min, p.dt_max);
  else
    dt_kernel<float><<<g, 256, 0, s>>>((const float *)p.dt, p.ds, p.dt_bias, p.dte, rows, p.H,
                                        p.softplus, p.dt_min, p.dt_max);
  return cudaGetLastError();
}

cudaError_t launch_conv_state_out(const PrefillPlan &p, cudaStream_t s) {
  if (!p.cso || p.W == 0) return cudaSuccess;
  const int elt = p.bf16 ? 2 : 4;
  const long long n = (long long)p.B * p.W * ((long long)p.conv_dim * elt / 16);
  const int g = grid_for(n, 256);
  if (p.bf16)
    conv_state_out_kernel<2><<<g, 256, 0, s>>>((const char *)p.xBC, p.xs * 2, (const char *)p.csi,
                                                (char *)p.cso, p.B, p.L, p.W, p.conv_dim);
  else
    conv_state_out_kernel<4><<<g, 256, 0, s>>>((const char *)p.xBC, p.xs * 4, (const char *)p.csi,
                                                (char *)p.cso, p.B, p.L, p.W, p.conv_dim);
  return cudaGetLastError();
}

cudaError_t launch_carry_only(const PrefillPlan &p, cudaStream_t s) {
  if (p.h_final && p.h_final != p.h0) {
    const long long n = (long long)p.B * p.H * p.P * p.N;
    carry_state_kernel<<<grid_for(n, 256), 256, 0, s>>>(p.h0, p.h_final, n);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return launch_conv_state_out(p, s);
}

}  // namespace ssd
