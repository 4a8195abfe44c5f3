// frontend.cu -- the scan's front end: causal depthwise conv1d (window W <= 4) + SiLU over
// the raw x|B|C channels, the effective time step softplus(dt_raw + dt_bias) with clamp, and
// the conv cache carried to the next call (the last W raw inputs, copied bit for bit).
//
// The conv of token t for channel c is silu(conv_b[c] + sum_k conv_w[c,k] * x[t-(W-1)+k, c]);
// inputs before the first token come from the incoming cache (row W-1 = the newest).  This is
// the Mamba-2 short convolution of window 4 in the Nemotron Nano 2 layers ("NVIDIA Nemotron
// Nano 2" summary, section "Method").
#include <algorithm>
#include <climits>
#include <type_traits>

#include "common.cuh"
#include "plan.h"

namespace ssd {
namespace {

constexpr int kConvTokens = 32;  // tokens per thread (sliding window kept in registers)

// One thread: 8 consecutive channels x kConvTokens consecutive tokens of one batch row.
// 16-byte vector loads along the channel dimension are coalesced across the warp.
// Channels [c_begin, c_begin + C_out) of the C-channel input are convolved; the output row
// holds C_out channels (fp32 for the CUDA-core path, bf16 for the tensor-core path).
template <typename T, typename OutT, int W, int TPT>
__global__ void __launch_bounds__(128) conv_silu_kernel(const T *__restrict__ xBC, long long xs,
                                                        const T *__restrict__ csi,
                                                        const T *__restrict__ w,
                                                        const T *__restrict__ bias,
                                                        OutT *__restrict__ u, int L, int C,
                                                        int c_begin, int C_out) {
  const int o8 = (blockIdx.x * blockDim.x + threadIdx.x) * 8;
  if (o8 >= C_out) return;
  const int c8 = c_begin + o8;
  const int b = blockIdx.z;
  const int t0 = blockIdx.y * TPT;
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
  const int t1 = min(L, t0 + TPT);
  // groups of 4 tokens: the 4 row loads are issued before any of them is used
  for (int tg = t0; tg < t1; tg += 4) {
    float cur[4][8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (tg + j < t1) load8(xrow + (long long)(tg + j) * xs + c8, cur[j]);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int t = tg + j;
      if (t >= t1) break;
      float out[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (W == 0) {
          out[i] = cur[j][i];
          continue;
        }
        // tap k multiplies time t-(W-1)+k: k = W-1 is cur, k = W-1-m is hist[3-m]
        float acc = bs[i] + wt[W > 0 ? W - 1 : 0][i] * cur[j][i];
#pragma unroll
        for (int m = 1; m < W; ++m) acc += wt[W - 1 - m][i] * hist[3 - m][i];
        out[i] = silu(acc);
      }
      store8(u + ((long long)b * L + t) * C_out + o8, out);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        hist[0][i] = hist[1][i];
        hist[1][i] = hist[2][i];
        hist[2][i] = cur[j][i];
      }
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

// Effective dt and its chunk-local inclusive prefix sum of dt*A, written head-major
// [B, H, Lpad] (Lpad = L rounded up to the 128-token chunk; padding has dt = 0 so the prefix
// stays flat).  One CTA: one 128-token chunk x 8 heads of one batch row.  Thread t reads the
// 8 heads of token t (16 bytes for bf16 when H % 8 == 0, else element by element), the tile
// is transposed through shared memory, and each warp scans two heads.
// The tile body: 128 threads (tid 0..127) and a 128 x 9 shared tile; every thread of the
// CTA must call it (it synchronises the CTA once), an inactive tile skips the work.
template <typename T>
__device__ __forceinline__ void dt_cumsum_tile(const T *__restrict__ dt, long long ds,
                                               const float *__restrict__ bias,
                                               const float *__restrict__ A, float *__restrict__ dte,
                                               float *__restrict__ cs, int L, int H, int Lpad, int sp,
                                               float lo, float hi, int c0, int h0, int b, int tid,
                                               float (*v)[9], bool active, const int *cu = nullptr,
                                               long long extent = LLONG_MAX, int *err = nullptr) {
  const int warp = tid / 32, lane = tid % 32;
  if (active) {
    const int tt = c0 + tid;
    float raw[8];
    const T *row = dt + (seq_base(cu, b, L) + tt) * ds + h0;
    L = seq_len(cu, b, L);  // this row's tokens; the tile's others are padding (dt = 0)
    if (tt < L && sizeof(T) == 2 && (H % 8) == 0 && (ds % 8) == 0) {
      load8(reinterpret_cast<const __nv_bfloat16 *>(row), raw);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) raw[j] = (tt < L && h0 + j < H) ? io<T>::ld(row + j) : 0.f;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j)
      v[tid][j] = (tt < L && h0 + j < H) ? effective_dt(raw[j], bias[h0 + j], sp, lo, hi) : 0.f;
  }
  __syncthreads();
  if (!active) return;
#pragma unroll
  for (int jj = 0; jj < 2; ++jj) {
    const int j = 2 * warp + jj, h = h0 + j;
    if (h >= H) break;
    const float a = A[h];
    float d[4], c[4];
    float run = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      d[i] = v[4 * lane + i][j];
      run += d[i] * a;
      c[i] = run;
    }
    float incl = run;  // inclusive scan of the per-lane totals
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    const float excl = incl - run;
    const long long base = ((long long)b * H + h) * Lpad + c0 + 4 * lane;
    if (in_bounds(base + 3, extent, err)) {  // dte and cs have the same extent
      *reinterpret_cast<float4 *>(dte + base) = make_float4(d[0], d[1], d[2], d[3]);
      *reinterpret_cast<float4 *>(cs + base) =
          make_float4(excl + c[0], excl + c[1], excl + c[2], excl + c[3]);
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(128) dt_cumsum_kernel(const T *__restrict__ dt, long long ds,
                                                         const float *__restrict__ bias,
                                                         const float *__restrict__ A,
                                                         float *__restrict__ dte,
                                                         float *__restrict__ cs, int L, int H,
                                                         int Lpad, int sp, float lo, float hi) {
  __shared__ float v[128][9];
  dt_cumsum_tile<T>(dt, ds, bias, A, dte, cs, L, H, Lpad, sp, lo, hi, blockIdx.x * 128, blockIdx.y * 8,
                    blockIdx.z, threadIdx.x, v, true);
}

// conv_state_out[b, k, :] = raw input of time L-W+k (from the incoming cache when negative).
// Copies 16-byte words without conversion, so the carried cache is bit-exact.
template <int ELT>
__device__ __forceinline__ void conv_state_out_range(const char *__restrict__ xBC, long long xs_bytes,
                                                     const char *__restrict__ csi, char *__restrict__ cso,
                                                     int B, int L, int W, int C, long long i0,
                                                     long long stride, const int *cu = nullptr) {
  const long long row_bytes = (long long)C * ELT;
  const long long vec_per_row = row_bytes / 16;
  const long long n = (long long)B * W * vec_per_row;
  for (long long i = i0; i < n; i += stride) {
    const long long v = i % vec_per_row;
    const int k = (int)((i / vec_per_row) % W);
    const int b = (int)(i / (vec_per_row * W));
    const int tau = seq_len(cu, b, L) - W + k;
    uint4 val = make_uint4(0, 0, 0, 0);
    if (tau >= 0)
      val = *reinterpret_cast<const uint4 *>(xBC + (seq_base(cu, b, L) + tau) * xs_bytes + v * 16);
    else if (csi)
      val = *reinterpret_cast<const uint4 *>(csi + ((long long)b * W + (W + tau)) * row_bytes + v * 16);
    *reinterpret_cast<uint4 *>(cso + ((long long)b * W + k) * row_bytes + v * 16) = val;
  }
}

template <int ELT>
__global__ void conv_state_out_kernel(const char *__restrict__ xBC, long long xs_bytes,
                                      const char *__restrict__ csi, char *__restrict__ cso, int B,
                                      int L, int W, int C, const int *cu) {
  conv_state_out_range<ELT>(xBC, xs_bytes, csi, cso, B, L, W, C,
                            blockIdx.x * (long long)blockDim.x + threadIdx.x,
                            (long long)gridDim.x * blockDim.x, cu);
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

// Many channels (the CUDA-core path converts every channel): 32 tokens per thread; few
// channels (B|C only): 8 tokens per thread, for enough threads to hide the load latency.
template <typename T, typename OutT, int W>
static void conv_launch(const PrefillPlan &p, OutT *out, int c_begin, int C_out, cudaStream_t s) {
  const int threads = 128;
  if (C_out >= 4096) {
    dim3 grid((C_out / 8 + threads - 1) / threads, (p.L + kConvTokens - 1) / kConvTokens, p.B);
    conv_silu_kernel<T, OutT, W, kConvTokens><<<grid, threads, 0, s>>>(
        (const T *)p.xBC, p.xs, (const T *)p.csi, (const T *)p.conv_w, (const T *)p.conv_b, out, p.L,
        p.conv_dim, c_begin, C_out);
  } else {
    dim3 grid((C_out / 8 + threads - 1) / threads, (p.L + 7) / 8, p.B);
    conv_silu_kernel<T, OutT, W, 8><<<grid, threads, 0, s>>>(
        (const T *)p.xBC, p.xs, (const T *)p.csi, (const T *)p.conv_w, (const T *)p.conv_b, out, p.L,
        p.conv_dim, c_begin, C_out);
  }
}

template <typename T, typename OutT>
static void conv_dispatch(const PrefillPlan &p, OutT *out, int c_begin, int C_out, cudaStream_t s) {
  switch (p.W) {
    case 0: conv_launch<T, OutT, 0>(p, out, c_begin, C_out, s); break;
    case 1: conv_launch<T, OutT, 1>(p, out, c_begin, C_out, s); break;
    case 2: conv_launch<T, OutT, 2>(p, out, c_begin, C_out, s); break;
    case 3: conv_launch<T, OutT, 3>(p, out, c_begin, C_out, s); break;
    default: conv_launch<T, OutT, 4>(p, out, c_begin, C_out, s); break;
  }
}

cudaError_t launch_conv_silu_f32(const PrefillPlan &p, cudaStream_t s) {
  if (p.bf16)
    conv_dispatch<__nv_bfloat16, float>(p, p.u, 0, p.conv_dim, s);
  else
    conv_dispatch<float, float>(p, p.u, 0, p.conv_dim, s);
  return cudaGetLastError();
}

// Conv + SiLU of the B and C channels into fp16 (the tensor-core scan's operand buffer).
// A streaming kernel: one thread owns 4 channels (one 8-byte load per row) over kBcTok
// tokens with the 4-row window kept in fp32 registers, and loads 8 rows ahead; few registers
// per thread keep several blocks per SM and tens of kilobytes of loads in flight.  The 3 rows
// before the first token come from the rows above (or the conv cache / zeros at t < 0).
constexpr int kBcTok = 16;
constexpr int kBcThreads = 256;

// SiLU(u) = u sigmoid(u) = h + h tanh(h) with h = u / 2, using the hardware tanh
// approximation (one special-function op instead of an exponential and a reciprocal).  Its
// error is of the order of the fp16 rounding that the result receives anyway.
__device__ __forceinline__ float silu_tanh(float u) {
  const float h = 0.5f * u;
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(h));
  return fmaf(h, t, h);
}

__device__ __forceinline__ void unpack4(const uint2 &r, float (&v)[4]) {
  v[0] = __uint_as_float(r.x << 16);
  v[1] = __uint_as_float(r.x & 0xFFFF0000u);
  v[2] = __uint_as_float(r.y << 16);
  v[3] = __uint_as_float(r.y & 0xFFFF0000u);
}

template <int W>
__device__ __forceinline__ void bc_conv_tile(const __nv_bfloat16 *__restrict__ xBC, long long xs,
                                             const __nv_bfloat16 *__restrict__ csi,
                                             const __nv_bfloat16 *__restrict__ w,
                                             const __nv_bfloat16 *__restrict__ bias,
                                             __half *__restrict__ out, int L, int conv_dim, int c_begin,
                                             int C_out, int bx, int by, int bz, const int *cu = nullptr,
                                             long long extent = LLONG_MAX, int *err = nullptr) {
  const int o4 = (bx * kBcThreads + threadIdx.x) * 4;
  if (o4 >= C_out) return;
  const int c4 = c_begin + o4;
  const int b = bz;
  const int t0 = by * kBcTok;
  const int t1 = min(seq_len(cu, b, L), t0 + kBcTok);
  if (t0 >= t1) return;  // past this row's tokens (a shorter sequence of a packed batch)
  const long long rb = seq_base(cu, b, L);
  const __nv_bfloat16 *xrow = xBC + rb * xs + c4;
  float wt[4][4], bs[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    bs[i] = bias ? __bfloat162float(bias[c4 + i]) : 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) wt[k][i] = (k < W) ? __bfloat162float(w[(long long)(c4 + i) * W + k]) : 0.f;
  }
  float x3[4], x2[4], x1[4];  // times t-3, t-2, t-1
  {
    uint2 hist[3];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      const int tau = t0 - 3 + j;
      if (W > 0 && tau >= 0) {
        hist[j] = *reinterpret_cast<const uint2 *>(xrow + (long long)tau * xs);
      } else if (csi && W > 0 && W + tau >= 0) {
        hist[j] = *reinterpret_cast<const uint2 *>(csi + ((long long)b * W + (W + tau)) * conv_dim + c4);
      } else {
        hist[j] = make_uint2(0u, 0u);
      }
    }
    unpack4(hist[0], x3);
    unpack4(hist[1], x2);
    unpack4(hist[2], x1);
  }
  // Rows in groups of 8; the common full tile runs without per-row bounds checks.
  auto group = [&](int tg, auto full_tag) {
    constexpr bool kFull = decltype(full_tag)::value;
    uint2 cur[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      cur[j] = (kFull || tg + j < t1) ? __ldcs(reinterpret_cast<const uint2 *>(xrow + (long long)(tg + j) * xs))
                                      : make_uint2(0u, 0u);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int t = tg + j;
      if (!kFull && t >= t1) break;
      float x0[4], r[4];
      unpack4(cur[j], x0);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (W == 0) {
          r[i] = x0[i];
        } else {
          // tap k multiplies time t-(W-1)+k
          const float xs4[4] = {x3[i], x2[i], x1[i], x0[i]};
          float acc = bs[i];
#pragma unroll
          for (int k = 0; k < W; ++k) acc = fmaf(wt[k][i], xs4[4 - W + k], acc);
          r[i] = silu_tanh(acc);
        }
        x3[i] = x2[i];
        x2[i] = x1[i];
        x1[i] = x0[i];
      }
      const __half2 h01 = __floats2half2_rn(r[0], r[1]), h23 = __floats2half2_rn(r[2], r[3]);
      const long long oi = (rb + t) * C_out + o4;
      if (in_bounds(oi + 3, extent, err))
        *reinterpret_cast<uint2 *>(out + oi) =
            make_uint2(*reinterpret_cast<const uint32_t *>(&h01), *reinterpret_cast<const uint32_t *>(&h23));
    }
  };
  if (t1 - t0 == kBcTok) {
    group(t0, std::true_type{});
    group(t0 + 8, std::true_type{});
  } else {
#pragma unroll 1
    for (int tg = t0; tg < t1; tg += 8) group(tg, std::false_type{});
  }
}

template <int W>
__global__ void __launch_bounds__(kBcThreads) bc_conv_kernel(const __nv_bfloat16 *__restrict__ xBC, long long xs,
                                                             const __nv_bfloat16 *__restrict__ csi,
                                                             const __nv_bfloat16 *__restrict__ w,
                                                             const __nv_bfloat16 *__restrict__ bias,
                                                             __half *__restrict__ out, int L, int conv_dim,
                                                             int c_begin, int C_out) {
  bc_conv_tile<W>(xBC, xs, csi, w, bias, out, L, conv_dim, c_begin, C_out, blockIdx.x, blockIdx.y, blockIdx.z);
}

// The tensor-core path's front end in one launch: dt + chunk prefix sums, the outgoing conv
// cache and the B/C conv, each CTA taking one role by its index (the latency-bound dt and
// cache CTAs first, so that they overlap the streaming B/C conv).  Registers are capped so
// that four CTAs share an SM: the launch is bound by the loads in flight, and three CTAs per
// SM (80 registers) measured 8-10 % slower.
struct FrontArgs {
  const __nv_bfloat16 *xBC, *dt, *csi, *conv_w, *conv_b;
  long long xs, ds;
  const float *dt_bias, *A;
  float *dte, *cs;
  __half *bc;
  __nv_bfloat16 *cso;
  int B, L, H, Lpad, conv_dim, d_inner, C_out, W, sp;
  float lo, hi;
  int n_dt, dt_tiles, dt_nch, dt_nhg, n_cso, gx, gy;
  const int *cu;  // packed variable-length batch offsets (device), or null
  long long bc_extent, dt_extent;  // elements of bc and of dte (= cs): the debug build's checks
  int *err;
};

template <int W>
__global__ void __launch_bounds__(kBcThreads, 4) front_tc_kernel(const FrontArgs f) {
  __shared__ float v[2][128][9];
  asm volatile("griddepcontrol.launch_dependents;");  // the scan may launch and set up now
  int j = blockIdx.x;
  if (j < f.n_dt) {  // two 128-thread dt tiles per CTA
    const int half = threadIdx.x >> 7, q = 2 * j + half;
    const bool active = q < f.dt_tiles;
    const int qq = active ? q : 0;
    const int cx = qq % f.dt_nch, hy = (qq / f.dt_nch) % f.dt_nhg, b = qq / (f.dt_nch * f.dt_nhg);
    dt_cumsum_tile<__nv_bfloat16>(f.dt, f.ds, f.dt_bias, f.A, f.dte, f.cs, f.L, f.H, f.Lpad, f.sp, f.lo,
                                  f.hi, cx * 128, hy * 8, b, threadIdx.x & 127, v[half], active, f.cu,
                                  f.dt_extent, f.err);
    return;
  }
  j -= f.n_dt;
  if (j < f.n_cso) {
    conv_state_out_range<2>((const char *)f.xBC, f.xs * 2, (const char *)f.csi, (char *)f.cso, f.B, f.L,
                            f.W, f.conv_dim, j * (long long)kBcThreads + threadIdx.x,
                            (long long)f.n_cso * kBcThreads, f.cu);
    return;
  }
  j -= f.n_cso;
  bc_conv_tile<W>(f.xBC, f.xs, f.csi, f.conv_w, f.conv_b, f.bc, f.L, f.conv_dim, f.d_inner, f.C_out,
                  j % f.gx, (j / f.gx) % f.gy, j / (f.gx * f.gy), f.cu, f.bc_extent, f.err);
}

cudaError_t launch_bc_conv_f16(const PrefillPlan &p, cudaStream_t s) {
  const int C_out = 2 * p.G * p.N;
  if (C_out % 4 || p.xs % 4 || p.conv_dim % 4 || p.d_inner % 4) {  // 8-byte accesses; else the generic kernel
    conv_dispatch<__nv_bfloat16, __half>(p, (__half *)p.bc, p.d_inner, C_out, s);
    return cudaGetLastError();
  }
  dim3 grid((C_out / 4 + kBcThreads - 1) / kBcThreads, (p.L + kBcTok - 1) / kBcTok, p.B);
  const auto *x = (const __nv_bfloat16 *)p.xBC;
  const auto *csi = (const __nv_bfloat16 *)p.csi;
  const auto *w = (const __nv_bfloat16 *)p.conv_w;
  const auto *bb = (const __nv_bfloat16 *)p.conv_b;
  __half *o = (__half *)p.bc;
  switch (p.W) {
    case 0: bc_conv_kernel<0><<<grid, kBcThreads, 0, s>>>(x, p.xs, csi, w, bb, o, p.L, p.conv_dim, p.d_inner, C_out); break;
    case 1: bc_conv_kernel<1><<<grid, kBcThreads, 0, s>>>(x, p.xs, csi, w, bb, o, p.L, p.conv_dim, p.d_inner, C_out); break;
    case 2: bc_conv_kernel<2><<<grid, kBcThreads, 0, s>>>(x, p.xs, csi, w, bb, o, p.L, p.conv_dim, p.d_inner, C_out); break;
    case 3: bc_conv_kernel<3><<<grid, kBcThreads, 0, s>>>(x, p.xs, csi, w, bb, o, p.L, p.conv_dim, p.d_inner, C_out); break;
    default: bc_conv_kernel<4><<<grid, kBcThreads, 0, s>>>(x, p.xs, csi, w, bb, o, p.L, p.conv_dim, p.d_inner, C_out); break;
  }
  return cudaGetLastError();
}

// False when the shapes need the separate front-end kernels (unaligned 8-byte B/C accesses).
bool front_tc_fusable(const PrefillPlan &p) {
  return p.bf16 && (2 * p.G * p.N) % 4 == 0 && p.xs % 4 == 0 && p.conv_dim % 4 == 0 && p.d_inner % 4 == 0 &&
         p.H % 8 == 0 && p.ds % 8 == 0;
}

cudaError_t launch_front_tc(const PrefillPlan &p, bool with_cso, cudaStream_t s) {
  FrontArgs f{};
  f.xBC = (const __nv_bfloat16 *)p.xBC; f.dt = (const __nv_bfloat16 *)p.dt;
  f.csi = (const __nv_bfloat16 *)p.csi; f.conv_w = (const __nv_bfloat16 *)p.conv_w;
  f.conv_b = (const __nv_bfloat16 *)p.conv_b; f.xs = p.xs; f.ds = p.ds; f.dt_bias = p.dt_bias; f.A = p.A;
  f.dte = p.dte_hm; f.cs = p.cs_hm; f.bc = (__half *)p.bc; f.cso = (__nv_bfloat16 *)p.cso;
  f.B = p.B; f.L = p.L; f.H = p.H; f.Lpad = p.Lpad; f.conv_dim = p.conv_dim; f.d_inner = p.d_inner;
  f.C_out = 2 * p.G * p.N; f.W = p.W; f.sp = p.softplus; f.lo = p.dt_min; f.hi = p.dt_max;
  f.cu = p.cu;
  f.bc_extent = checked_extent(p, p.rows * 2LL * p.G * p.N);
  f.dt_extent = checked_extent(p, (long long)p.B * p.H * p.Lpad);
  f.err = p.err;
  f.dt_nch = p.Lpad / 128; f.dt_nhg = (p.H + 7) / 8; f.dt_tiles = f.dt_nch * f.dt_nhg * p.B;
  f.n_dt = (f.dt_tiles + 1) / 2;
  const long long ncso = (with_cso && p.cso && p.W > 0) ? (long long)p.B * p.W * ((long long)p.conv_dim * 2 / 16) : 0;
  f.n_cso = ncso ? (int)std::min<long long>((ncso + kBcThreads - 1) / kBcThreads, 64) : 0;
  f.gx = (f.C_out / 4 + kBcThreads - 1) / kBcThreads; f.gy = (p.L + kBcTok - 1) / kBcTok;
  const long long blocks = (long long)f.n_dt + f.n_cso + (long long)f.gx * f.gy * p.B;
  switch (p.W) {
    case 0: front_tc_kernel<0><<<(unsigned)blocks, kBcThreads, 0, s>>>(f); break;
    case 1: front_tc_kernel<1><<<(unsigned)blocks, kBcThreads, 0, s>>>(f); break;
    case 2: front_tc_kernel<2><<<(unsigned)blocks, kBcThreads, 0, s>>>(f); break;
    case 3: front_tc_kernel<3><<<(unsigned)blocks, kBcThreads, 0, s>>>(f); break;
    default: front_tc_kernel<4><<<(unsigned)blocks, kBcThreads, 0, s>>>(f); break;
  }
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

cudaError_t launch_dt_cumsum(const PrefillPlan &p, float *dte, float *cs, int Lpad, cudaStream_t s) {
  dim3 grid(Lpad / 128, (p.H + 7) / 8, p.B);
  if (p.bf16)
    dt_cumsum_kernel<__nv_bfloat16><<<grid, 128, 0, s>>>((const __nv_bfloat16 *)p.dt, p.ds, p.dt_bias,
                                                          p.A, dte, cs, p.L, p.H, Lpad, p.softplus,
                                                          p.dt_min, p.dt_max);
  else
    dt_cumsum_kernel<float><<<grid, 128, 0, s>>>((const float *)p.dt, p.ds, p.dt_bias, p.A, dte, cs,
                                                  p.L, p.H, Lpad, p.softplus, p.dt_min, p.dt_max);
  return cudaGetLastError();
}

cudaError_t launch_conv_state_out(const PrefillPlan &p, cudaStream_t s) {
  if (!p.cso || p.W == 0) return cudaSuccess;
  const int elt = p.bf16 ? 2 : 4;
  const long long n = (long long)p.B * p.W * ((long long)p.conv_dim * elt / 16);
  const int g = grid_for(n, 256);
  if (p.bf16)
    conv_state_out_kernel<2><<<g, 256, 0, s>>>((const char *)p.xBC, p.xs * 2, (const char *)p.csi,
                                                (char *)p.cso, p.B, p.L, p.W, p.conv_dim, p.cu);
  else
    conv_state_out_kernel<4><<<g, 256, 0, s>>>((const char *)p.xBC, p.xs * 4, (const char *)p.csi,
                                                (char *)p.cso, p.B, p.L, p.W, p.conv_dim, p.cu);
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
