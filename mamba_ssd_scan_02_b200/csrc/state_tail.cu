// state_tail.cu -- the final state's last chunks in fp32.
//
// The tensor-core scan carries the state in fp32 but multiplies fp16 operands, and the final
// state's largest entries often come from a few recent tokens, whose products are not
// averaged over many terms.  So this pass computes, in fp32 from the raw inputs, what the last
// kTailChunks chunks (at most 256 tokens) of the sequence's last segment add to the final
// state, starting from a zero state:
//   per chunk:  dH <- e^{cs_Q} dH + sum_s e^{cs_Q - cs_s} dt_s x_s B_s^T
// with x_s, B_s the causal conv1d + SiLU of the raw channels (history from the incoming conv
// cache before token 0) and dt_s, cs_s the chunk-local prefix sums of dt*A already computed
// for the scan.  The output scan leaves the state entering those chunks, and a fold sets
// h = e^{sum of their cs_Q} h + dH.
//
// It needs only the front end's outputs, so it runs on a side stream beside the output scan:
// on the SMs the scan leaves free, a few persistent CTAs work through the (head, batch row)
// items.
//
// Per item, a CTA of 512 threads computes every tail token's weight w_s = e^{cs_Q - cs_s}
// dt_s; per chunk it copies the chunk's raw rows of its 64 x channels and its group's 128 B
// channels (plus 3 history rows) into shared memory with asynchronous 16-byte copies (all in
// flight together).  Per 64 tokens, threads 0..383 then run the conv + SiLU, one channel and
// 32 tokens each (a sliding window over the staged rows), writing fp32 outputs with the x
// channels already multiplied by w_s; after one barrier all 16 warps apply those tokens'
// rank-1 updates.  The staging of one chunk (about 100 KB of shared memory in all) lets two
// CTAs share an SM, so that one's copies overlap the other's arithmetic.  For those, warp w owns state rows 16 (w >> 2) .. +15 and
// columns 32 (w & 3) .. +31, and a lane a 4 x 4 block, so one token costs a warp two
// conflict-free 16-byte shared loads (4 x values, 4 B values) and eight paired FMAs.
#include <algorithm>

#include "common.cuh"
#include "plan.h"

namespace ssd {
namespace {

constexpr int kTailThreads = 512;
constexpr int kTailMax = 256;                      // tokens in the tail at most (2 chunks)
constexpr int kTailCh = kHeadDim + kDState;        // 192 channels: the head's x, the group's B
constexpr int kConvThreads = 2 * kTailCh;          // two 32-token strips per channel
constexpr int kStep = 64;                          // tokens per conv + update round
constexpr int kRawRows = 128 + 3;                  // one chunk and its 3 history rows
constexpr size_t kRawBytes = (size_t)kRawRows * kTailCh * 2;           // bf16 raw rows
constexpr size_t kOutBytes = (size_t)kStep * kTailCh * 4;              // one round's fp32 outputs
constexpr size_t kTailSmem = kRawBytes + kOutBytes + kTailMax * 4;     // + token weights
static_assert(2 * kTailSmem + 2048 <= 228 * 1024, "two tail CTAs per SM");
static_assert(kTailThreads == 16 * 32 && kHeadDim == 64 && kDState == 128, "warp tiling assumes 64 x 128");

// 16-byte global -> shared copy that zero-fills when src_bytes is 0 (the source is not read).
__device__ __forceinline__ void cp_async16(void *dst, const void *src, int src_bytes) {
  const unsigned d = static_cast<unsigned>(__cvta_generic_to_shared(dst));
  const size_t g = __cvta_generic_to_global(src);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(g), "r"(src_bytes) : "memory");
}

__global__ void __launch_bounds__(kTailThreads, 2) state_tail_kernel(
    const __nv_bfloat16 *__restrict__ xBC, long long xs, const __nv_bfloat16 *__restrict__ conv_w,
    const __nv_bfloat16 *__restrict__ conv_b, const __nv_bfloat16 *__restrict__ csi,
    const float *__restrict__ dte, const float *__restrict__ cs, float *__restrict__ dh_out,
    float *__restrict__ dec_out, int L, int B, int H, int hpg, int conv_dim, int d_inner, int W,
    int Lpad, int t_tail_uniform, const int *__restrict__ cu) {
  extern __shared__ __align__(16) unsigned char tsm[];
  __nv_bfloat16 *raw = reinterpret_cast<__nv_bfloat16 *>(tsm);       // [kRawRows][192]
  float *uo = reinterpret_cast<float *>(tsm + kRawBytes);             // [64][192]
  float *ws = reinterpret_cast<float *>(tsm + kRawBytes + kOutBytes);  // [256]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int p0 = 16 * (warp >> 2) + 4 * (lane >> 3), n0 = 32 * (warp & 3) + 4 * (lane & 7);
  // conv role: channel ch (column of raw / uo), 32-token strip hf of each round; tap j reads
  // time t-3+j
  const bool conv_thread = tid < kConvThreads;
  const int ch = tid % kTailCh, hf = tid / kTailCh;
  for (int item = blockIdx.x; item < B * H; item += gridDim.x) {
    const int h = item % H, b = item / H, g = h / hpg;
    // this row's tokens and tail (a packed variable-length batch has one segment per sequence,
    // its tail the last two chunks of the sequence)
    const int Lb = seq_len(cu, b, L);
    int t_tail = t_tail_uniform;
    if (cu) {
      const int nckb = (Lb + 127) / 128;
      t_tail = 128 * (nckb > kTailChunks ? nckb - kTailChunks : 0);
    }
    const int ntok = Lb - t_tail;  // 0 .. kTailMax
    const __nv_bfloat16 *xrow = xBC + seq_base(cu, b, L) * xs;
    const float *csr = cs + ((long long)b * H + h) * Lpad;
    const float *dtr = dte + ((long long)b * H + h) * Lpad;

    // token weights w_s = e^{cs_Q - cs_s} dt_s, cs_Q the prefix at the end of the token's chunk
    // (chunk-local prefix sums; the padding past L has dt = 0, so the prefix stays flat there)
    for (int i = tid; i < ntok; i += kTailThreads)
      ws[i] = __expf(csr[t_tail + (i & ~127) + 127] - csr[t_tail + i]) * dtr[t_tail + i];
    float acc[16];  // acc[4 i + j] = dH[p0 + i][n0 + j]
#pragma unroll
    for (int j = 0; j < 16; ++j) acc[j] = 0.f;
    const int cch = ch < kHeadDim ? h * kHeadDim + ch : d_inner + g * kDState + (ch - kHeadDim);
    float wt[4] = {0.f, 0.f, 0.f, 0.f}, bias = 0.f;
    if (conv_thread && W > 0) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int k = j - (4 - W);
        if (k >= 0) wt[j] = __bfloat162float(conv_w[(long long)cch * W + k]);
      }
      if (conv_b) bias = __bfloat162float(conv_b[cch]);
    }

    for (int c0 = 0; c0 < ntok; c0 += 128) {  // chunks of the tail (t_tail is chunk-aligned)
      const int n = min(128, ntok - c0);
      // raw rows of times t_tail+c0-3 .. t_tail+c0+n-1: 24 16-byte pieces per row (8 of x,
      // 16 of B); the previous chunk's readers finished at the barrier that ended it
      for (int i = tid; i < (n + 3) * 24; i += kTailThreads) {
        const int r = i / 24, v = i % 24, tau = t_tail + c0 - 3 + r;
        const int c = v < 8 ? h * kHeadDim + 8 * v : d_inner + g * kDState + 8 * (v - 8);
        const void *src = xBC;  // not read when zero-filling
        int bytes = 0;
        if (tau >= 0) {
          src = xrow + (long long)tau * xs + c; bytes = 16;
        } else if (csi && W + tau >= 0) {
          src = csi + ((long long)b * W + (W + tau)) * conv_dim + c; bytes = 16;
        }
        cp_async16(raw + r * kTailCh + 8 * v, src, bytes);
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
      asm volatile("cp.async.wait_all;" ::: "memory");
      __syncthreads();
      const float decay = __expf(csr[t_tail + c0 + 127]);
#pragma unroll
      for (int j = 0; j < 16; ++j) acc[j] *= decay;
      for (int h0 = 0; h0 < n; h0 += kStep) {
        const int m = min(kStep, n - h0);
        if (conv_thread) {
          const int s_lo = h0 + hf * (kStep / 2), s_hi = min(s_lo + kStep / 2, n);
          if (s_lo < s_hi) {
            const __nv_bfloat16 *col = raw + s_lo * kTailCh + ch;  // raw row of time t-3 for s_lo
            float xm3 = __bfloat162float(col[0]), xm2 = __bfloat162float(col[kTailCh]),
                  xm1 = __bfloat162float(col[2 * kTailCh]);
            const bool is_x = ch < kHeadDim;
#pragma unroll 8
            for (int s = s_lo; s < s_hi; ++s) {
              const float x0 = __bfloat162float(raw[(s + 3) * kTailCh + ch]);
              float v = x0;
              if (W > 0) v = silu(fmaf(wt[0], xm3, fmaf(wt[1], xm2, fmaf(wt[2], xm1, fmaf(wt[3], x0, bias)))));
              uo[(s - h0) * kTailCh + ch] = is_x ? v * ws[c0 + s] : v;
              xm3 = xm2; xm2 = xm1; xm1 = x0;
            }
          }
        }
        __syncthreads();  // the round's conv outputs are ready
#pragma unroll 4
        for (int s = 0; s < m; ++s) {
          const float4 xv = *reinterpret_cast<const float4 *>(uo + s * kTailCh + p0);  // weighted x
          const float4 bv = *reinterpret_cast<const float4 *>(uo + s * kTailCh + kHeadDim + n0);
          const float2 b01 = make_float2(bv.x, bv.y), b23 = make_float2(bv.z, bv.w);
          const float xa[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 a2 = make_float2(xa[i], xa[i]);
            const float2 lo = __ffma2_rn(a2, b01, make_float2(acc[4 * i], acc[4 * i + 1]));
            const float2 hi = __ffma2_rn(a2, b23, make_float2(acc[4 * i + 2], acc[4 * i + 3]));
            acc[4 * i] = lo.x; acc[4 * i + 1] = lo.y; acc[4 * i + 2] = hi.x; acc[4 * i + 3] = hi.y;
          }
        }
        __syncthreads();  // the outputs (and raw rows, weights) are consumed before they are rewritten
      }
    }
    if (tid == 0) {  // decay over the tail's chunks
      float sum = 0.f;
      for (int c0 = 0; c0 < ntok; c0 += 128) sum += csr[t_tail + c0 + 127];
      dec_out[(long long)b * H + h] = __expf(sum);
    }
    float *dblk = dh_out + (((long long)b * H + h) * kHeadDim + p0) * kDState + n0;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      *reinterpret_cast<float4 *>(dblk + i * kDState) = make_float4(acc[4 * i], acc[4 * i + 1], acc[4 * i + 2], acc[4 * i + 3]);
  }  // item
}

}  // namespace

// One tail item (a head of a batch row) costs about as much as this many chunks of the scan.
constexpr int kItemChunks = 8;

// The tail starts at chunk nck-kTailChunks of the last segment (its first chunk when it has
// fewer).  Grid: two CTAs on each SM the output scan (one CTA per SM, n_seg x H x B of them)
// leaves free, when they finish all items within the scan's time; otherwise two per SM of the
// whole GPU, up to one CTA per item.
cudaError_t launch_state_tail(const PrefillPlan &p, cudaStream_t s) {
  static_assert(kTailChunks * 128 <= kTailMax, "tail longer than the staging buffers");
  if (!p.tail_dh || p.L == 0) return cudaSuccess;
  const int t_b = (p.n_seg - 1) * p.seg_len;
  const int nck = (p.L - t_b + 127) / 128;
  const int t_tail = t_b + 128 * (nck > kTailChunks ? nck - kTailChunks : 0);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long items = (long long)p.B * p.H;
  const long long scan_ctas = (long long)p.n_seg * p.H * p.B;
  const long long seg_chunks = (p.seg_len + 127) / 128;
  const long long free_sms = sms - scan_ctas;
  const long long need = (items * kItemChunks + seg_chunks - 1) / seg_chunks;  // CTAs to keep pace
  // two CTAs per SM
  long long grid = 2 * (free_sms >= need && free_sms >= 1 ? free_sms : sms);
  if (grid > items) grid = items;
  cudaError_t e = set_smem_attr(state_tail_kernel, kTailSmem, s);
  if (e != cudaSuccess) return e;
  state_tail_kernel<<<(unsigned)grid, kTailThreads, kTailSmem, s>>>(
      (const __nv_bfloat16 *)p.xBC, p.xs, (const __nv_bfloat16 *)p.conv_w, (const __nv_bfloat16 *)p.conv_b,
      (const __nv_bfloat16 *)p.csi, p.dte_hm, p.cs_hm, p.tail_dh, p.tail_dec, p.L, p.B, p.H, p.hpg,
      p.conv_dim, p.d_inner, p.W, p.Lpad, t_tail, p.cu);
  return cudaGetLastError();
}

}  // namespace ssd
