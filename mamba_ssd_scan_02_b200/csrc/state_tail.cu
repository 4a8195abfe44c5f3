// state_tail.cu -- the final state's last chunks at fp32 accuracy.
//
// The tensor-core scan carries the state in fp32 but multiplies fp16 operands, and the final
// state's largest entries often come from a few recent tokens, whose products are not
// averaged over many terms.  So this pass computes, from the raw inputs, what the last
// kTailChunks chunks (at most 256 tokens) of the sequence's last segment add to the final
// state, starting from a zero state:
//   per chunk:  dH <- e^{cs_Q} dH + sum_s e^{cs_Q - cs_s} dt_s x_s B_s^T
// with x_s, B_s the causal conv1d + SiLU of the raw channels (history from the incoming conv
// cache before token 0) and dt_s, cs_s the chunk-local prefix sums of dt*A already computed
// for the scan.  Unrolled over the (at most two) chunks, dH = sum_s w_s x_s B_s^T with
// w_s = e^{cs_Q(s) - cs_s + cs_Q of the later chunk, if any} dt_s.  The output scan leaves the
// state entering those chunks, and a fold sets h = e^{sum of their cs_Q} h + dH.
//
// It needs only the front end's outputs, so it runs on a side stream beside the output scan,
// on the SMs the scan leaves free: persistent CTAs (one per SM) work through items of up to
// four heads of one group and batch row, which share the group's B channels.  When the scan
// leaves too few SMs free (many short sequences, large batches), it runs after the scan on
// all SMs instead and folds its part into the state the scan left (h = e^{...} h + dH), with
// no dH buffer and no fold pass.
//
// Per item the CTA computes every tail token's weight w_s per head; then, per 64 tokens (a
// round), it copies the raw rows of the heads' x channels and the group's B channels (plus 3
// history rows) into shared memory with asynchronous 16-byte copies (the next round's copies,
// or the next item's first, run during this round), and each thread runs the conv + SiLU in
// fp32 for two adjacent channels over 16 tokens, multiplies the x channels by w_s, and splits
// each value v into fp16 parts, v = hi + lo + e with hi = fp16(v), lo = fp16(v - hi) and
// |e| <= 2^-22 |v| (plus an absolute 2^-25 where lo falls below fp16's normal range), written
// into 128-byte-swizzled operand tiles.  One thread then issues the round's update on the
// tensor cores, one MMA per 16 tokens and product for all the item's heads (N = 64 per head),
// into a tensor-memory accumulator (128 lanes = state column n, 64 columns per head), as three
// fp16 products with fp32 accumulation:
//   dH^T += B_hi^T X_hi + B_hi^T X_lo + B_lo^T X_hi
// (the dropped lo*lo term is below 2^-22 of the product), which keeps the update at fp32
// accuracy.  Sixteen warps finally read the accumulator and store dH (or fold it).
#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "plan.h"
#include "tc_ptx.cuh"

namespace ssd {
namespace {

using namespace tc;

constexpr int kTailThreads = 768;
constexpr int kTailHeads = 4;                        // heads per item
constexpr int kTailMax = 256;                        // tokens in the tail at most (2 chunks)
constexpr int kRound = 64;                           // tokens per round (the MMAs' K)
constexpr int kRawCh = kTailHeads * kHeadDim + kDState;  // 384 staged channels: x of 4 heads, B
constexpr int kPairs = kRawCh / 2;                   // a thread converts two adjacent channels
constexpr int kStrips = kTailThreads / kPairs;       // 4 strips of 16 tokens per round
constexpr int kStripTok = kRound / kStrips;
constexpr int kRawRows = kRound + 3;                 // a round's rows and their 3 history rows
// shared memory, bytes from a 1024-aligned base (the operand tiles need the alignment for the
// 128-byte swizzle)
constexpr uint32_t kRawBuf = (uint32_t)kRawRows * kRawCh * 2;  // bf16 raw rows, double-buffered
constexpr uint32_t OFF_AH = 103424;                  // B^T high parts: 2 boxes of 64 tokens x 64 n
constexpr uint32_t OFF_AL = OFF_AH + 16384;          // B^T low parts
constexpr uint32_t OFF_XH = OFF_AL + 16384;          // w x high parts: 4 boxes of 64 tokens x 64 p
constexpr uint32_t OFF_XL = OFF_XH + 32768;          // w x low parts
constexpr uint32_t OFF_WS = OFF_XL + 32768;          // token weights [4 heads][256] fp32
constexpr uint32_t OFF_BAR = OFF_WS + kTailHeads * kTailMax * 4;
constexpr uint32_t OFF_MISC = OFF_BAR + 8;           // [0] TMEM base, [1] abort flag, [2] drain flag
constexpr uint32_t OFF_DEC = OFF_MISC + 16;          // the item's heads' tail decays [4] fp32
constexpr uint32_t kTailSmem = OFF_DEC + 16 + 1024;  // + room to align the base
constexpr uint32_t kTailCols = kTailHeads * kHeadDim;  // the accumulator: 64 columns per head
static_assert(2 * kRawBuf <= OFF_AH && OFF_AH % 1024 == 0 && OFF_XH % 1024 == 0 && OFF_XL % 1024 == 0,
              "tile layout");
static_assert(kTailSmem <= 232448, "shared memory budget");
static_assert(kPairs * kStrips == kTailThreads && kPairs % 32 == 0 && kStripTok % 8 == 0,
              "warps are uniform in role and strip");
static_assert(kHeadDim == 64 && kDState == 128, "tiles assume 64 x 128");

// 16-byte global -> shared copy that zero-fills when src_bytes is 0 (the source is not read).
__device__ __forceinline__ void cp_async16(void *dst, const void *src, int src_bytes) {
  const unsigned d = static_cast<unsigned>(__cvta_generic_to_shared(dst));
  const size_t g = __cvta_generic_to_global(src);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(g), "r"(src_bytes) : "memory");
}

// SiLU(a) = a / (1 + e^{-a}) = a / (1 + 2^{-a log2(e)}), two values at a time, from the
// hardware base-2 exponential and reciprocal approximations (each within a few units in the
// last place of fp32): about 2^-21 relative error, well inside the pass's fp32 accuracy (the
// final state's error is dominated by the fp32 prefix sums of dt*A it shares with the scan)
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float2 silu2(float2 a) {
  const float2 t = __fmul2_rn(a, make_float2(-1.4426950408889634f, -1.4426950408889634f));
  const float2 d = __fadd2_rn(make_float2(1.f, 1.f), make_float2(ex2_approx(t.x), ex2_approx(t.y)));
  return __fmul2_rn(a, make_float2(rcp_approx(d.x), rcp_approx(d.y)));
}

__device__ __forceinline__ float2 ld_bf16x2(const __nv_bfloat16 *p) {
  const uint32_t u = *reinterpret_cast<const uint32_t *>(p);
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}

// One item: heads h0 .. h0+nh-1 of group g of batch row b, and its tail tokens.
struct TailItem {
  int b, g, nh, h0, t_tail, ntok;
  long long base;  // token row of the sequence's first token
};

__device__ __forceinline__ TailItem tail_item(int item, int nq, int G, int hpg, int L, int t_tail_uniform,
                                              const int *cu) {
  TailItem it;
  const int q = item % nq, bg = item / nq;
  it.g = bg % G;
  it.b = bg / G;
  it.nh = min(kTailHeads, hpg - kTailHeads * q);
  it.h0 = it.g * hpg + kTailHeads * q;
  // a packed variable-length batch has one segment per sequence, its tail the last two chunks
  // of the sequence
  const int Lb = seq_len(cu, it.b, L);
  int t_tail = t_tail_uniform;
  if (cu) {
    const int nckb = (Lb + 127) / 128;
    t_tail = 128 * (nckb > kTailChunks ? nckb - kTailChunks : 0);
  }
  it.t_tail = t_tail;
  it.ntok = Lb - t_tail;  // 0 .. kTailMax
  it.base = seq_base(cu, it.b, L);
  return it;
}

// Asynchronous copies of round r's raw rows (times t_tail + 64r - 3 ..) of the item's x and B
// channels into raw[row][384] (x of head i at columns 64i.., B at 256..), as one commit group.
// A row is 48 pieces of 16 bytes; thread tid copies piece tid % 48 of rows tid / 48, +16, ...
constexpr int kPieces = kRawCh / 8;
constexpr int kRowsPerPass = kTailThreads / kPieces;
static_assert(kTailThreads % kPieces == 0, "whole rows per pass");
__device__ __forceinline__ void tail_stage(const TailItem &it, int r, __nv_bfloat16 *raw,
                                           const __nv_bfloat16 *__restrict__ xBC, long long xs,
                                           const __nv_bfloat16 *__restrict__ csi, int W, int conv_dim,
                                           int d_inner, int tid) {
  const int tok0 = r * kRound;
  const int rows = min(kRawRows, it.ntok - tok0 + 3);
  const int v = tid % kPieces;
  const bool vx = v < 8 * kTailHeads;
  if (vx && (v >> 3) >= it.nh) {  // a head the item does not have
    asm volatile("cp.async.commit_group;" ::: "memory");
    return;
  }
  const int rc = 8 * v;  // raw column: x of head v / 8, then B
  const int c = vx ? (it.h0 + (v >> 3)) * kHeadDim + 8 * (v & 7) : d_inner + it.g * kDState + 8 * (v - 8 * kTailHeads);
  const __nv_bfloat16 *xcol = xBC + it.base * xs + c;
  for (int k = tid / kPieces; k < rows; k += kRowsPerPass) {
    const int tau = it.t_tail + tok0 - 3 + k;
    const void *src = xBC;  // not read when zero-filling
    int bytes = 0;
    if (tau >= 0) {
      src = xcol + (long long)tau * xs; bytes = 16;
    } else if (csi && W + tau >= 0) {
      src = csi + ((long long)it.b * W + (W + tau)) * conv_dim + c; bytes = 16;
    }
    cp_async16(raw + k * kRawCh + rc, src, bytes);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}

__global__ void __launch_bounds__(kTailThreads, 1) state_tail_kernel(
    const __nv_bfloat16 *__restrict__ xBC, long long xs, const __nv_bfloat16 *__restrict__ conv_w,
    const __nv_bfloat16 *__restrict__ conv_b, const __nv_bfloat16 *__restrict__ csi,
    const float *__restrict__ dte, const float *__restrict__ cs, float *__restrict__ dh_out,
    float *__restrict__ dec_out, int L, int B, int H, int G, int hpg, int conv_dim, int d_inner, int W,
    int Lpad, int t_tail_uniform, const int *__restrict__ cu, int *err, float *h_fold,
    long long dh_extent, long long dec_extent) {
  extern __shared__ unsigned char tsm_raw[];
  // aligned by an offset from the shared array itself (not through an integer), so that the
  // compiler keeps every access derived from it in the shared address space
  unsigned char *tsm = tsm_raw + ((1024u - (smem_u32(tsm_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(tsm);
  float *ws = reinterpret_cast<float *>(tsm + OFF_WS);  // [4][256]
  float *decs = reinterpret_cast<float *>(tsm + OFF_DEC);  // [4]
  uint32_t *misc = reinterpret_cast<uint32_t *>(tsm + OFF_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 1);
  volatile int *drain_flag = reinterpret_cast<volatile int *>(misc + 2);
  const uint32_t bar = sb + OFF_BAR;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // conv role: channel pair `pair` (0-127: x of head pair / 32, 128-191: B), 16-token strip
  const int pair = tid % kPairs, strip = tid / kPairs;
  const bool is_x = pair < kTailHeads * 32;
  const int xhead = pair >> 5;                        // x pairs: the head within the item
  const int rcol = 2 * pair;                          // raw column (x of head i at 64i, B at 256)
  const int tcol = is_x ? 2 * (pair & 31) : (2 * (pair - 128)) & 63;  // column within its box
  unsigned char *hi_tile = tsm + (is_x ? OFF_XH + (uint32_t)xhead * 8192u
                                       : OFF_AH + (uint32_t)((2 * (pair - 128)) >> 6) * 8192u);
  // byte offset of this thread's 4 bytes in a swizzled row r, by r mod 8 (16-byte chunk
  // c / 8 of row r sits at chunk (c / 8) ^ (r % 8))
  uint32_t loff[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) loff[u] = ((uint32_t)(((tcol >> 3) ^ u) & 7) << 4) + (uint32_t)(tcol & 7) * 2u;
  if (tid == 0) {
    mbar_init(bar, 1);
    *abort_flag = 0;
    *drain_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(sb + OFF_MISC, kTailCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  const int nq = (hpg + kTailHeads - 1) / kTailHeads;
  const int items = B * G * nq;
  uint32_t phase = 0;   // parity of the next commit's phase
  uint32_t gr = 0;      // rounds staged so far (raw buffer gr % 2)
  bool staged = false;  // the current item's first round is already staged
  bool failed = false;  // a bounded wait ran out (uniform across the CTA)

  for (int item = blockIdx.x; item < items && !failed; item += gridDim.x) {
    const TailItem it = tail_item(item, nq, G, hpg, L, t_tail_uniform, cu);
    const int nr = (it.ntok + kRound - 1) / kRound;
    if (!staged && nr > 0)
      tail_stage(it, 0, reinterpret_cast<__nv_bfloat16 *>(tsm + (gr & 1) * kRawBuf), xBC, xs, csi, W,
                 conv_dim, d_inner, tid);
    staged = false;
    const int nch = (it.ntok + 127) / 128;
    // token weights (the previous item's readers finished at its last barrier)
    for (int i = tid; i < it.nh * kTailMax; i += kTailThreads) {
      const int hh = i >> 8, t = i & (kTailMax - 1);
      if (t < it.ntok) {
        const long long row = ((long long)it.b * H + it.h0 + hh) * Lpad + it.t_tail;
        const float later = (nch == 2 && t < 128) ? cs[row + 255] : 0.f;
        ws[i] = __expf(cs[row + (t & ~127) + 127] - cs[row + t] + later) * dte[row + t];
      }
    }
    const bool active = !is_x || xhead < it.nh;
    const int cch = is_x ? (it.h0 + xhead) * kHeadDim + 2 * (pair & 31) : d_inner + it.g * kDState + 2 * (pair - 128);
    float2 wt[4], bias = make_float2(0.f, 0.f);  // tap j multiplies time t-3+j
#pragma unroll
    for (int j = 0; j < 4; ++j) wt[j] = make_float2(0.f, 0.f);
    if (W > 0 && active) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int k = j - (4 - W);
        if (k >= 0)
          wt[j] = make_float2(__bfloat162float(conv_w[(long long)cch * W + k]),
                              __bfloat162float(conv_w[(long long)(cch + 1) * W + k]));
      }
      if (conv_b) bias = make_float2(__bfloat162float(conv_b[cch]), __bfloat162float(conv_b[cch + 1]));
    }
    const uint32_t idesc = idesc_f16(128, kHeadDim * it.nh, true, true, kFmtF16);

    for (int r = 0; r < nr && !failed; ++r, ++gr) {
      const __nv_bfloat16 *raw = reinterpret_cast<const __nv_bfloat16 *>(tsm + (gr & 1) * kRawBuf);
      asm volatile("cp.async.wait_all;" ::: "memory");
      __syncthreads();  // this round's rows landed; the other buffer's last readers are done
      {  // the next round's rows (or the next item's first) into the other buffer
        __nv_bfloat16 *nxt = reinterpret_cast<__nv_bfloat16 *>(tsm + ((gr + 1) & 1) * kRawBuf);
        if (r + 1 < nr) {
          tail_stage(it, r + 1, nxt, xBC, xs, csi, W, conv_dim, d_inner, tid);
        } else if (item + (int)gridDim.x < items) {
          const TailItem nx = tail_item(item + gridDim.x, nq, G, hpg, L, t_tail_uniform, cu);
          if (nx.ntok > 0) {
            tail_stage(nx, 0, nxt, xBC, xs, csi, W, conv_dim, d_inner, tid);
            staged = true;
          }
        }
      }
      // the previous round's products read the tiles that this round rewrites
      if (r > 0) {
        mbar_wait(bar, phase, abort_flag, err);
        phase ^= 1u;
      }
      const int tok0 = r * kRound, s_lo = strip * kStripTok;
      if (active) {  // conv + SiLU of 16 tokens of two channels; rows past the tail are zero
        const __nv_bfloat16 *colp = raw + s_lo * kRawCh + rcol;  // raw row of time t-3 for s_lo
        const int nvalid = it.ntok - tok0 - s_lo;
        const float *wsr = ws + xhead * kTailMax + tok0 + s_lo;
        unsigned char *hrow = hi_tile + (uint32_t)s_lo * 128u;  // row s_lo of this thread's hi tile
        // the strip's tokens, all present (kFull) or checked one by one; kX: x channels (times
        // w_s); kConv: a causal conv (W > 0) -- compile-time, so the unrolled loop has no branch
        auto strip_tokens = [&](auto full_tag, auto x_tag, auto conv_tag) {
          constexpr bool kFull = decltype(full_tag)::value, kX = decltype(x_tag)::value,
                         kConv = decltype(conv_tag)::value;
          constexpr uint32_t kLo = kX ? OFF_XL - OFF_XH : OFF_AL - OFF_AH;  // lo tile after the hi one
          float2 xm3 = ld_bf16x2(colp), xm2 = ld_bf16x2(colp + kRawCh), xm1 = ld_bf16x2(colp + 2 * kRawCh);
#pragma unroll 8
          for (int i = 0; i < kStripTok; ++i) {
            uint32_t hw = 0u, lw = 0u;
            if (kFull || i < nvalid) {
              const float2 x0 = ld_bf16x2(colp + (i + 3) * kRawCh);
              float2 v = x0;
              if constexpr (kConv)
                v = silu2(__ffma2_rn(wt[3], x0, __ffma2_rn(wt[2], xm1, __ffma2_rn(wt[1], xm2, __ffma2_rn(wt[0], xm3, bias)))));
              if constexpr (kX) {
                const float w = wsr[i];
                v = __fmul2_rn(v, make_float2(w, w));
              }
              const __half2 hi = __float22half2_rn(v);
              const float2 hf = __half22float2(hi);
              const __half2 lo = __float22half2_rn(make_float2(v.x - hf.x, v.y - hf.y));
              hw = *reinterpret_cast<const uint32_t *>(&hi);
              lw = *reinterpret_cast<const uint32_t *>(&lo);
              xm3 = xm2; xm2 = xm1; xm1 = x0;
            }
            unsigned char *q = hrow + (uint32_t)i * 128u + loff[i & 7];
            *reinterpret_cast<uint32_t *>(q) = hw;
            *reinterpret_cast<uint32_t *>(q + kLo) = lw;
          }
        };
        const bool full = nvalid >= kStripTok;
        auto by_shape = [&](auto x_tag) {
          if (W > 0) {
            if (full) strip_tokens(std::true_type{}, x_tag, std::true_type{});
            else strip_tokens(std::false_type{}, x_tag, std::true_type{});
          } else {
            if (full) strip_tokens(std::true_type{}, x_tag, std::false_type{});
            else strip_tokens(std::false_type{}, x_tag, std::false_type{});
          }
        };
        if (is_x) by_shape(std::true_type{});
        else by_shape(std::false_type{});
      }
      fence_proxy_async();  // the tiles' generic writes, visible to the tensor cores
      if (__syncthreads_or(*abort_flag != 0)) {
        failed = true;
        break;
      }
      if (tid == 0) {  // dH^T (128 n x 64 nh p) += the round's three fp16 products
        tc_fence_after();
        const uint64_t ah = smem_desc_sw128(sb + OFF_AH, 8192, 1024), al = smem_desc_sw128(sb + OFF_AL, 8192, 1024);
        const uint64_t xh = smem_desc_sw128(sb + OFF_XH, 8192, 1024), xl = smem_desc_sw128(sb + OFF_XL, 8192, 1024);
#pragma unroll
        for (int j = 0; j < kRound / 16; ++j) {
          // K step j: 16 token rows of 128 bytes further (the descriptors' address field is in
          // 16-byte units and every address here lies below 256 KB, so the add stays in it)
          const uint64_t o = (uint64_t)((j * 2048) >> 4);
          mma_f16_ss(tmem, ah + o, xh + o, idesc, (r > 0 || j > 0) ? 1u : 0u);
          mma_f16_ss(tmem, ah + o, xl + o, idesc, 1u);
          mma_f16_ss(tmem, al + o, xh + o, idesc, 1u);
        }
        mma_commit(bar);
      }
    }
    if (failed) break;
    if (nr > 0) {  // the last round's products
      mbar_wait(bar, phase, abort_flag, err);
      phase ^= 1u;
      tc_fence_after();
      if (__syncthreads_or(*abort_flag != 0)) {
        failed = true;
        break;
      }
    }
    if (tid < it.nh) {  // decay over the tail's chunks
      const float *csr = cs + ((long long)it.b * H + it.h0 + tid) * Lpad + it.t_tail;
      float sum = 0.f;
      for (int c0 = 0; c0 < it.ntok; c0 += 128) sum += csr[c0 + 127];
      decs[tid] = __expf(sum);
      const long long di = (long long)it.b * H + it.h0 + tid;
      if (!h_fold && in_bounds(di, dec_extent, err)) dec_out[di] = decs[tid];
    }
    if (h_fold) __syncthreads();  // the decays, for the fold below
    // dH of head warp / 4, lanes (state columns n) 32 (warp % 4) ..: into dh_out, or folded
    // into the state the scan left in h_fold (h = dec h + dH)
    if (warp < 4 * kTailHeads && (warp >> 2) < it.nh) {
      const int hh = warp >> 2, qd = warp & 3, nn = 32 * qd + lane;
      const long long d0 = ((long long)it.b * H + it.h0 + hh) * kHeadDim * kDState + nn;  // dst's index
      float *dst = (h_fold ? h_fold : dh_out) + d0;
      const float dec = decs[hh];
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {  // 16 columns (p) at a time
        float a[16];
        if (nr > 0) {
          tmem_ld16(tmem + ((uint32_t)(32 * qd) << 16) + (uint32_t)(kHeadDim * hh + 16 * c), a);
          tmem_ld_wait();
        }
        if (nr == 0) {
#pragma unroll
          for (int i = 0; i < 16; ++i) a[i] = 0.f;
        }
        float *q = dst + 16 * c * kDState;  // a warp stores 32 consecutive n
        const long long qi = d0 + 16 * c * kDState;  // q's index
        if (h_fold) {  // 16 loads in flight, then the stores
          float hv[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) hv[i] = q[i * kDState];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (in_bounds(qi + i * kDState, dh_extent, err)) q[i * kDState] = fmaf(dec, hv[i], a[i]);
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (in_bounds(qi + i * kDState, dh_extent, err)) q[i * kDState] = a[i];
        }
      }
    }
    tc_fence_before();
    __syncthreads();  // the accumulator is read before the next item's first product
    tc_fence_after();
  }  // item
  // after a wait ran out, the products it waited for may still be in flight: wait for them
  // (within 0.1 s, on a flag of its own, since the abort flag ends a wait at once) before the
  // accumulator is freed; copies still in flight land in this CTA's own shared memory
  if (failed && tid == 0) mbar_wait(bar, phase ^ 1u, drain_flag, nullptr, 100000000ull);
  asm volatile("cp.async.wait_all;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTailCols);
  }
}

}  // namespace

namespace {

// One tail item (four heads of a batch row) costs about as much as this many chunks of the scan.
constexpr int kItemChunks = 4;

struct TailGrid {
  long long items, free_sms;
  int sms;
  bool beside;
};

// The output scan takes one SM per CTA (n_seg x H x B of them); the tail pass fits beside it
// when the SMs it leaves free finish all tail items within the scan's time.
TailGrid tail_grid(const PrefillPlan &p) {
  TailGrid g{};
  int dev = 0;
  g.sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&g.sms, cudaDevAttrMultiProcessorCount, dev);
  g.items = (long long)p.B * p.G * ((p.hpg + kTailHeads - 1) / kTailHeads);
  const long long scan_ctas = (long long)p.n_seg * p.H * p.B;
  const long long seg_chunks = (p.seg_len + 127) / 128;
  g.free_sms = g.sms - scan_ctas;
  const long long need = (g.items * kItemChunks + seg_chunks - 1) / seg_chunks;  // CTAs to keep pace
  g.beside = g.free_sms >= need && g.free_sms >= 1;
  return g;
}

}  // namespace

bool tail_beside_scan(const PrefillPlan &p) { return tail_grid(p).beside; }

// The tail starts at chunk nck-kTailChunks of the last segment (its first chunk when it has
// fewer).  Grid: one CTA on each SM the scan leaves free when the pass runs beside it, else one
// per SM of the whole GPU; at most one CTA per item.
cudaError_t launch_state_tail(const PrefillPlan &p, bool fold_in, cudaStream_t s) {
  static_assert(kTailChunks * 128 <= kTailMax, "tail longer than the weight buffer");
  if (!p.tail_dh || p.L == 0) return cudaSuccess;
  if (p.xs % 8 || p.conv_dim % 8 || p.d_inner % 8) return cudaErrorInvalidValue;  // 16-byte copies
  if (fold_in && !p.h_final) return cudaErrorInvalidValue;
  const int t_b = (p.n_seg - 1) * p.seg_len;
  const int nck = (p.L - t_b + 127) / 128;
  const int t_tail = t_b + 128 * (nck > kTailChunks ? nck - kTailChunks : 0);
  const TailGrid tg = tail_grid(p);
  long long grid = tg.beside ? tg.free_sms : tg.sms;
  if (grid > tg.items) grid = tg.items;
  cudaError_t e = set_smem_attr(state_tail_kernel, kTailSmem, s);
  if (e != cudaSuccess) return e;
  state_tail_kernel<<<(unsigned)grid, kTailThreads, kTailSmem, s>>>(
      (const __nv_bfloat16 *)p.xBC, p.xs, (const __nv_bfloat16 *)p.conv_w, (const __nv_bfloat16 *)p.conv_b,
      (const __nv_bfloat16 *)p.csi, p.dte_hm, p.cs_hm, p.tail_dh, p.tail_dec, p.L, p.B, p.H, p.G, p.hpg,
      p.conv_dim, p.d_inner, p.W, p.Lpad, t_tail, p.cu, p.err, fold_in ? p.h_final : nullptr,
      checked_extent(p, (long long)p.B * p.H * kHeadDim * kDState), checked_extent(p, (long long)p.B * p.H));
  return cudaGetLastError();
}

}  // namespace ssd
