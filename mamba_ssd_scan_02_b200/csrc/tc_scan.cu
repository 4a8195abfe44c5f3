// tc_scan.cu -- chunked SSD scan on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// One CTA per (segment, head, batch row) walks its segment's 128-token chunks in order and
// keeps the head's P x N = 64 x 128 state on chip.  For chunk k with cs = chunk-local prefix
// sums of dt*A (cs_Q = cs at the last token), the Mamba-2 scan becomes four dense fp16
// contractions with fp32 accumulation in tensor memory:
//   MMA1  S     = C . B^T                    M=128 (t) N=128 (s) K=128 (n)   -> TMEM S[k%2]
//   mask  S~    = S o (e^{cs_t - cs_s} dt_s [s <= t]) + D_h I   (CUDA cores; written back
//                 into the same TMEM columns as packed fp16)
//   MMA2  Yi    = S~ . X                     M=128 (t) N=64 (p)  K=128 (s)   (A from TMEM)
//   MMA3  Ys    = C . h_{k-1}^T              M=128 (t) N=64 (p)  K=128 (n)
//   MMA4  dH^T  = B^T . (w o X), w_s = e^{cs_Q - cs_s} dt_s   M=128 (n) N=64 (p) K=128 (s)
// then y_t = Yi + e^{cs_t} Ys (the D x skip is folded into the diagonal of S~) and
// h_k = e^{cs_Q} h_{k-1} + dH, kept in fp32 in TMEM (an fp16 copy feeds MMA3 of chunk k+1).
// This is the token recurrence h_t = e^{dt_t A} h_{t-1} + dt_t x_t B_t^T, y_t = h_t C_t + D x_t
// regrouped by chunk; every exponent is a difference cs_t - cs_s <= 0 or is split at a
// 32-token block boundary where both factors stay below e^60 (else computed directly).
// In the last chunk of a segment w o X is applied as fp16 hi + lo parts (a second MMA4), so
// a segment's final state carries the rounding of B only: its largest entries come from the
// newest tokens, whose products are not averaged over many terms.  The sequence's own final
// state goes further: in tail mode the output pass leaves the state entering the last two
// chunks, and a separate fp32 pass (state_tail.cu) adds those chunks' contribution.
//
// Warp roles (640 threads): warp 0 issues TMA loads (B and C tiles of the group, the head's
// raw x rows with a 3-token halo, per-chunk dt and prefix sums), warp 1 allocates TMEM and
// issues each MMA group as soon as its inputs are ready, warps 2-9 compute the x channels
// (causal conv1d + SiLU) in place into w o X and into X, warps 10-15 turn S into S~, warps
// 16-19 update the state (kept in fp32 in TMEM), refresh its fp16 copy and write y.
// X, w o X, S (with Yi in its upper half), Ys and the B/C stages are double-buffered, so each
// role can run a chunk ahead of the next.  Hand-offs use mbarriers (TMA transaction counts,
// tcgen05.commit, thread arrivals); every wait is bounded and a timeout aborts the CTA
// cleanly and latches SSD_ERR_TIMEOUT.
//
// Operands are fp16 (the conv outputs B, C, x are O(10) in the workloads, far inside the fp16
// range; 11 significant bits keep the chunked products within the bf16-input tolerance).
// Shared-memory operand layouts use the 128-byte swizzle: B/C tiles are two TMA boxes of
// 64 channels x 128 tokens (K-major for MMA1/MMA3, M-major for MMA4); X, w o X and the fp16
// state copy are 128-byte rows (N-major B operands).
#include <cudaTypedefs.h>

#include <type_traits>

#include "common.cuh"
#include "plan.h"
#include "tc_ptx.cuh"

// Optional timeline marks for one CTA (compiled only with -DSSD_TC_TRACE): device time of
// each role's steps per chunk, read back by a measurement tool.
#ifdef SSD_TC_TRACE
__device__ unsigned long long g_tc_trace[256 * 16];
#define TC_MARK(k, e)                                                                         \
  do {                                                                                        \
    if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && (k) < 256)                   \
      g_tc_trace[(k) * 16 + (e)] = ssd::tc::globaltimer();                                    \
  } while (0)
extern "C" int ssd_tc_trace_read(unsigned long long *out) {
  return cudaMemcpyFromSymbol(out, g_tc_trace, sizeof(g_tc_trace)) == cudaSuccess ? 0 : 1;
}
#else
#define TC_MARK(k, e) \
  do {                \
  } while (0)
#endif

namespace ssd {
namespace {

using namespace tc;

constexpr int QC = 128;              // tokens per chunk
constexpr int kThreadsTC = 640;       // 20 warps
constexpr int kConvWarps = 8;          // see conv_index()
constexpr int kTokPerConvWarp = QC / kConvWarps;  // 16
constexpr uint32_t kTile = 16384;    // one 128-row x 128-byte operand box
// per-stage layout (bytes)
constexpr uint32_t OFF_C = 0;                 // C tile: channels 0-63 | 64-127
constexpr uint32_t OFF_B = 2 * kTile;         // B tile
constexpr uint32_t OFF_DT = 4 * kTile;        // dt[128] fp32
constexpr uint32_t OFF_CS = OFF_DT + 512;     // cs[128] fp32
constexpr uint32_t kStage = 4 * kTile + 1024;  // 66560 = 65 * 1024
// CTA layout.  w o X[b] (two buffers, chunk k uses b = k % 2) first receives by TMA the
// chunk's raw bf16 x rows for times t0-3 .. t0+127 (131 rows of this head's 64 channels); the
// conv overwrites row s with the w o X row s and writes X row s into X[b].  The raw tile thus
// waits only for MMA4 of chunk k-2 (which frees w o X[b]), not for MMA2, which comes later.
constexpr uint32_t kXBuf = 17 * 1024;           // 131 rows of 128 bytes, padded
constexpr uint32_t kRawRows = QC + 3;
constexpr uint32_t OFF_X = 2 * kStage;              // X[2]  [s][p] fp16, 16 KB each
constexpr uint32_t OFF_XW = OFF_X + 2 * kTile;      // w o X [2][s][p] fp16 (raw x rows first)
constexpr uint32_t OFF_H = OFF_XW + 2 * kXBuf;      // h copy [n][p] fp16, 16 KB
constexpr uint32_t OFF_CF = OFF_H + kTile;          // column factors, 128 fp32
constexpr uint32_t OFF_CSM = OFF_CF + 512;          // the mask's copies of cs and dt
constexpr uint32_t OFF_DTM = OFF_CSM + 512;
constexpr uint32_t OFF_BAR = OFF_DTM + 512;
// Barriers.  Every event that can recur before its consumer has observed the previous
// occurrence has one barrier per buffer, so that a parity test never sees two phases at once.
enum {
  BAR_FULL0, BAR_FULL1,        // stage k % 2 loaded (TMA)
  BAR_EMPTY0, BAR_EMPTY1,      // stage k % 2 released (conv, mask, state warps + MMA commit)
  BAR_FULLX0, BAR_FULLX1,      // raw x of chunk k in w o X[k % 2] (TMA)
  BAR_XFREE0, BAR_XFREE1,      // X[k % 2] read by MMA2 of chunk k
  BAR_SREADY0, BAR_SREADY1,    // S of chunk k in TMEM (MMA1)
  BAR_STREADY0, BAR_STREADY1,  // S~ of chunk k in TMEM (mask warps)
  BAR_XREADY0, BAR_XREADY1,    // X and w o X of chunk k written (conv warps)
  BAR_XWFREE0, BAR_XWFREE1,    // w o X[k % 2] read by MMA4 of chunk k
  BAR_DHREADY,                 // dH of chunk k in TMEM (MMA4)
  BAR_DHFREE,                  // dH of chunk k read by the state warps
  BAR_HTFREE,                  // h tile (h_{k-1}) read by MMA3 of chunk k
  BAR_HREADY,                  // h tile holds h_k (state warps)
  BAR_YREADY0, BAR_YREADY1,    // Yi and Ys of chunk k in TMEM (MMA2 commit)
  BAR_YFREE0, BAR_YFREE1,      // Yi and Ys of chunk k read by the output warps
  BAR_XLOREADY,                // low part of w o X of the last chunk written
  BAR_DONE,
  kNumBars
};
constexpr uint32_t OFF_MISC = OFF_BAR + 8 * 32;   // [0] TMEM base, [1] abort flag
constexpr uint32_t kSmemUsed = OFF_MISC + 16;
constexpr uint32_t kSmemAlloc = kSmemUsed + 1024;  // room to align the base to 1024 bytes
static_assert(kNumBars <= 32, "barrier slots");
static_assert(kSmemAlloc <= 232448, "shared memory budget");
static_assert(OFF_X % 1024 == 0 && kXBuf % 1024 == 0 && OFF_XW % 1024 == 0 && OFF_H % 1024 == 0,
              "swizzle alignment");
static_assert(kRawRows * 128 <= kXBuf, "raw x tile fits its buffer");

// TMEM columns (fp32 accumulators, 128 lanes).  S[b] (chunk k uses b = k % 2) first holds S;
// the mask rewrites it as packed fp16 S~ in columns 0-63, and MMA2 then accumulates Yi into
// columns 64-127 (whose S values the mask has read).  Ys is double-buffered likewise.
constexpr uint32_t TM_S0 = 0, TM_S1 = 128, TM_YS0 = 256, TM_YS1 = 320, TM_DH = 384, TM_H = 448,
                   TM_COLS = 512;  // TM_H: the fp32 state h^T (row n, column p)
constexpr uint32_t TM_YI_OFF = 64;  // Yi within S[b]

constexpr uint32_t IDESC_S = idesc_f16(128, 128, false, false, kFmtF16);  // C K-major, B K-major
constexpr uint32_t IDESC_YS = idesc_f16(128, 64, false, true, kFmtF16);   // C K-major, h N-major
constexpr uint32_t IDESC_YI = idesc_f16(128, 64, false, true, kFmtF16);   // S~ (TMEM), X N-major
constexpr uint32_t IDESC_DH = idesc_f16(128, 64, true, true, kFmtF16);    // B M-major, wX N-major

struct TcArgs {
  int B, L, H, G, hpg, conv_dim, Lpad, W, seg_len;
  const __nv_bfloat16 *xBC;
  long long xs;
  const __nv_bfloat16 *csi, *conv_w, *conv_b;
  const float *dte, *cs, *D;
  const float *h_init;     // initial state (per segment when h_init_seg > 0) or null = 0
  long long h_init_seg;
  float *h_out;            // final state destination or null
  long long h_out_seg;
  int tail_chunks;         // > 0: instead of the final state, the last segment writes the state
                           // before its last tail_chunks chunks (an fp32 pass finishes it)
  float *seg_decay;        // [n_seg, B, H] total decay per segment, or null
  __nv_bfloat16 *y;        // output (no gate) ...
  long long ys;
  __half *yh;              // ... or fp16 pre-norm output [rows, d_inner] when the gated norm
                           //     follows (its pass reads it with z)
  int d_inner;
  int *err;
  unsigned long long wait_ns;  // limit of every bounded wait
  int debug_skip_chunk;        // test hook (-1 = off): the producer stops before loading this
                               // chunk's stage, so its consumers' bounded waits run out
  long long y_extent, h_extent;  // elements of the y (or yh) and h_out buffers (index checks
                               // of the debug build)
  const int *cu;               // packed variable-length batch: sequence b is token rows
                               // cu[b] .. cu[b+1]-1 (the tensor maps then have one batch row
                               // of all the tokens); null: row b*L + t
};

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&v);
}
__device__ __forceinline__ uint32_t pack_f16(float a, float b) {
  __half2 v = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&v);
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
  __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162 *>(&u);
  return __bfloat1622float2(v);
}

// A group-uniform bounded wait: one leader thread waits on the mbarrier, then the group
// syncs on its named barrier, which ORs every thread's view of the abort flag so that all of
// them take the same branch.
__device__ __forceinline__ bool wg_wait(uint32_t bar, uint32_t parity, bool leader, int nb,
                                        volatile int *abort_flag, int *err, uint64_t limit_ns,
                                        int nthreads = 128) {
  if (leader) mbar_wait(bar, parity, abort_flag, err, limit_ns);
  return !named_bar_or(nb, nthreads, *abort_flag != 0);
}

// ---- MMA issue (single thread) ---------------------------------------------------------
// The issuing thread shares its SM sub-partition with busy warps, so each group costs it as
// few instructions as possible: fully unrolled, with the shared-memory descriptors built once
// and advanced by adding to their start-address field (bits 0-13, in 16-byte units; every
// operand lies below 256 KB, so the add never carries out of the low word).
__device__ __forceinline__ uint64_t desc_adv(uint64_t d, uint32_t bytes) {
  const uint32_t lo = static_cast<uint32_t>(d) + (bytes >> 4);
  return (d & 0xFFFFFFFF00000000ull) | lo;
}
// K step j of a K-major 128-row operand stored as two 64-column boxes: 32 bytes per step
// within a box, the second box after four steps.
__device__ __forceinline__ constexpr uint32_t kmajor_step(int j) { return (j >> 2) * kTile + (j & 3) * 32; }

__device__ __forceinline__ void issue_S(uint32_t stage, uint32_t tS) {
  const uint64_t a0 = smem_desc_sw128(stage + OFF_C, 16, 1024), b0 = smem_desc_sw128(stage + OFF_B, 16, 1024);
#pragma unroll
  for (int j = 0; j < 8; ++j)
    mma_f16_ss(tS, desc_adv(a0, kmajor_step(j)), desc_adv(b0, kmajor_step(j)), IDESC_S, j > 0);
}
__device__ __forceinline__ void issue_Ys(uint32_t stage, uint32_t hbase, uint32_t tYs) {
  const uint64_t a0 = smem_desc_sw128(stage + OFF_C, 16, 1024), b0 = smem_desc_sw128(hbase, 8192, 1024);
#pragma unroll
  for (int j = 0; j < 8; ++j)
    mma_f16_ss(tYs, desc_adv(a0, kmajor_step(j)), desc_adv(b0, j * 2048), IDESC_YS, j > 0);
}
// S~ in TMEM: 16 fp16 of K per MMA = 8 columns
__device__ __forceinline__ void issue_Yi(uint32_t tSt, uint32_t xbase, uint32_t tYi) {
  const uint64_t b0 = smem_desc_sw128(xbase, 8192, 1024);
#pragma unroll
  for (int j = 0; j < 8; ++j) mma_f16_ts(tYi, tSt + 8 * j, desc_adv(b0, j * 2048), IDESC_YI, j > 0);
}
__device__ __forceinline__ void issue_dH(uint32_t stage, uint32_t xwbase, uint32_t tDH, bool acc) {
  const uint64_t a0 = smem_desc_sw128(stage + OFF_B, kTile, 1024), b0 = smem_desc_sw128(xwbase, 8192, 1024);
#pragma unroll
  for (int j = 0; j < 8; ++j)
    mma_f16_ss(tDH, desc_adv(a0, j * 2048), desc_adv(b0, j * 2048), IDESC_DH, (j > 0 || acc) ? 1u : 0u);
}

// Conv warps: 2-9, two on each SM sub-partition (warp % 4), the issuer's included: spreading
// them evenly measured faster than keeping the issuer's sub-partition free of them.
__device__ __forceinline__ int conv_index(int warp) { return warp >= 2 && warp < 10 ? warp - 2 : -1; }

// Row r (128 bytes) of a 128-byte-swizzled tile: 16-byte chunk c sits at chunk c ^ (r & 7).
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return (uint32_t)row * 128u + ((uint32_t)(chunk ^ (row & 7)) << 4);
}

// fp16 copy of state columns p = 32*half .. 32*half+31 of row n into the h tile
__device__ __forceinline__ void write_h_tile(unsigned char *smem, const float (&hr)[32], int n, int half) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint4 v = make_uint4(pack_f16(hr[8 * c + 0], hr[8 * c + 1]), pack_f16(hr[8 * c + 2], hr[8 * c + 3]),
                         pack_f16(hr[8 * c + 4], hr[8 * c + 5]), pack_f16(hr[8 * c + 6], hr[8 * c + 7]));
    *reinterpret_cast<uint4 *>(smem + OFF_H + swz(n, 4 * half + c)) = v;
  }
}

// kStateOnly: the states-only pass (no y); kConv: the x channels have a causal conv (W > 0),
// a compile-time switch so that the token loops carry no branch on it.
template <bool kStateOnly, bool kConv>
__global__ void __launch_bounds__(kThreadsTC, 1)
    ssd_scan_tc_kernel(const __grid_constant__ CUtensorMap tm_bc,
                       const __grid_constant__ CUtensorMap tm_x, const TcArgs a) {
  extern __shared__ unsigned char smem_raw[];
  // aligned by an offset from the shared array itself (not through an integer), so that the
  // compiler keeps every access derived from it in the shared address space
  unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int seg = blockIdx.x, h = blockIdx.y, b = blockIdx.z, g = h / a.hpg;
  const int t_begin = seg * a.seg_len;
  const int t_end = min(seq_len(a.cu, b, a.L), t_begin + a.seg_len);
  // TMA coordinates of this row's token t: (t + tma_t0, batch tma_b)
  const int tma_t0 = a.cu ? a.cu[b] : 0, tma_b = a.cu ? 0 : b;
  const int nck = t_end > t_begin ? (t_end - t_begin + QC - 1) / QC : 0;
  const int last = nck - 1;
  // The last chunk's exact path (fp32 SiLU, split-precision w o X) serves only the final
  // state, which the full pass never takes from here: with a final state requested it runs
  // in tail mode (an fp32 pass recomputes the last chunks), and otherwise nothing reads it.
  // So only the states-only pass compiles it.
  constexpr bool exact_last = kStateOnly;
  const uint64_t lim = a.wait_ns;
  const uint32_t bar0 = sb + OFF_BAR;
#define BAR(i) (bar0 + 8u * (uint32_t)(i))
  uint32_t *misc = reinterpret_cast<uint32_t *>(smem + OFF_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 1);

  if (tid == 0) {
    for (int i = 0; i < kNumBars; ++i) {
      uint32_t cnt = 1;
      if (i == BAR_EMPTY0 || i == BAR_EMPTY1) cnt = kStateOnly ? 3 : 4;  // + mask warps
      if (i == BAR_XREADY0 || i == BAR_XREADY1 || i == BAR_XLOREADY) cnt = kConvWarps;
      mbar_init(BAR(i), cnt);
    }
    *abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_bc);
    prefetch_tmap(&tm_x);
  }
  if (warp == 1) {
    tmem_alloc(sb + OFF_MISC, TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    // Raw x rows of chunk k go to w o X[k % 2] once MMA4 of chunk k-2 has released it; the
    // B/C tiles, dt and prefix sums go to stage k % 2 once chunk k-2's consumers released it.
    if (lane == 0) {
      int k = 0, nx = 0, nbc = 0;
      for (; k < nck; ++k) {
        const int xb = k & 1, st = k & 1;
        const int t0 = t_begin + k * QC;
        if (k >= 2 && !mbar_wait(BAR(BAR_XWFREE0 + xb), ((k >> 1) - 1) & 1, abort_flag, a.err, lim)) break;
        mbar_arrive_expect_tx(BAR(BAR_FULLX0 + xb), kRawRows * 128);
        tma_load_3d(sb + OFF_XW + xb * kXBuf, &tm_x, h * 64, tma_t0 + t0 - 3, tma_b, BAR(BAR_FULLX0 + xb));
        ++nx;
        if (a.debug_skip_chunk == k) break;  // test hook: stage k never arrives (see TcArgs)
        if (k >= 2 && !mbar_wait(BAR(BAR_EMPTY0 + st), ((k >> 1) - 1) & 1, abort_flag, a.err, lim)) break;
        // the stage holds the front end's outputs: the kernel may have been launched before
        // the front end finished (programmatic dependent launch), and waits for it here; the
        // raw x rows above are the caller's input, complete before the front end started
        if (k == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
        const uint32_t sst = sb + st * kStage;
        const uint32_t full = BAR(BAR_FULL0 + st);
        TC_MARK(k, 12);
        mbar_arrive_expect_tx(full, (kStateOnly ? 2 * kTile : 4 * kTile) + 1024);
        const int cB = g * 128, cC = a.G * 128 + g * 128;
        if (!kStateOnly) {
          tma_load_3d(sst + OFF_C, &tm_bc, cC, tma_t0 + t0, tma_b, full);
          tma_load_3d(sst + OFF_C + kTile, &tm_bc, cC + 64, tma_t0 + t0, tma_b, full);
        }
        tma_load_3d(sst + OFF_B, &tm_bc, cB, tma_t0 + t0, tma_b, full);
        tma_load_3d(sst + OFF_B + kTile, &tm_bc, cB + 64, tma_t0 + t0, tma_b, full);
        const long long hoff = ((long long)b * a.H + h) * a.Lpad + t0;
        bulk_load(sst + OFF_DT, a.dte + hoff, 512, full);
        bulk_load(sst + OFF_CS, a.cs + hoff, 512, full);
        ++nbc;
      }
      // every load issued must land before the CTA may exit
      int never_abort = 0;
      for (int j = (nx >= 2 ? nx - 2 : 0); j < nx; ++j)
        mbar_wait(BAR(BAR_FULLX0 + (j & 1)), (j >> 1) & 1, &never_abort, a.err);
      for (int j = (nbc >= 2 ? nbc - 2 : 0); j < nbc; ++j)
        mbar_wait(BAR(BAR_FULL0 + (j & 1)), (j >> 1) & 1, &never_abort, a.err);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    // Issues each chunk's four MMA groups as soon as their inputs are ready, whatever the
    // order, so that no group waits behind another one that is still blocked:
    //   MMA1 S(j)   stage j loaded; S[j % 2] free (MMA2 of chunk j-2 issued, its output read)
    //   MMA4 dH(j)  X(j) and w o X(j) written; dH of chunk j-1 read by the state warps
    //   MMA3 Ys(j)  after MMA1(j); h_{j-1} in the h tile
    //   MMA2 Yi(j)  after MMA3(j) and MMA4(j); S~(j) written by the mask warps
    // A commit after each group signals its consumers; stage j is released by a commit after
    // the last of MMA1/MMA3/MMA4 of chunk j.  Polling sleeps briefly when nothing is ready and
    // gives up (abort + SSD_ERR_TIMEOUT) after ~2 s without progress.
    if (lane == 0) {
      int nS = kStateOnly ? nck : 0, nD = 0, nYs = kStateOnly ? nck : 0, nYi = kStateOnly ? nck : 0;
      auto stage_done = [&](int j) {  // all readers of stage j issued?
        return nD > j && (kStateOnly || (nS > j && nYs > j));
      };
      uint64_t t_prog = globaltimer();
      uint32_t nap = 32;  // sleep between polls: doubles up to 256 ns while nothing is ready
      bool ok = true;
      while (ok && (nD < nck || nYi < nck)) {
        bool prog = false;
        if (nYi < nck && nYi < nYs && nYi < nD && mbar_test(BAR(BAR_STREADY0 + (nYi & 1)), (nYi >> 1) & 1)) {
          const int j = nYi;
          tc_fence_after();
          TC_MARK(j, 11);
          const uint32_t tS = tmem + ((j & 1) ? TM_S1 : TM_S0);
          issue_Yi(tS, sb + OFF_X + (j & 1) * kTile, tS + TM_YI_OFF);
          mma_commit(BAR(BAR_YREADY0 + (j & 1)));
          mma_commit(BAR(BAR_XFREE0 + (j & 1)));
          ++nYi;
          prog = true;
        }
        if (nYs < nck && nYs < nS && mbar_test(BAR(BAR_HREADY), nYs & 1)) {
          const int j = nYs;
          tc_fence_after();
          TC_MARK(j, 9);
          issue_Ys(sb + (j & 1) * kStage, sb + OFF_H, tmem + ((j & 1) ? TM_YS1 : TM_YS0));
          mma_commit(BAR(BAR_HTFREE));
          ++nYs;
          if (stage_done(j)) mma_commit(BAR(BAR_EMPTY0 + (j & 1)));
          prog = true;
        }
        if (nD < nck && (kStateOnly || nD < nS) &&
            mbar_test(BAR(BAR_XREADY0 + (nD & 1)), (nD >> 1) & 1) &&
            (nD == 0 || mbar_test(BAR(BAR_DHFREE), (nD - 1) & 1)) &&
            (nD != last || !exact_last || mbar_test(BAR(BAR_XLOREADY), 0)) &&
            (!kStateOnly || mbar_test(BAR(BAR_FULL0 + (nD & 1)), (nD >> 1) & 1))) {
          const int j = nD;
          tc_fence_after();
          TC_MARK(j, 8);
          const uint32_t sst = sb + (j & 1) * kStage;
          issue_dH(sst, sb + OFF_XW + (j & 1) * kXBuf, tmem + TM_DH, false);
          // last chunk: the low part of w o X (in the other w o X buffer) for the final state
          if (j == last && exact_last) issue_dH(sst, sb + OFF_XW + ((j + 1) & 1) * kXBuf, tmem + TM_DH, true);
          mma_commit(BAR(BAR_XWFREE0 + (j & 1)));
          mma_commit(BAR(BAR_DHREADY));
          if (kStateOnly) mma_commit(BAR(BAR_XFREE0 + (j & 1)));
          ++nD;
          if (stage_done(j)) mma_commit(BAR(BAR_EMPTY0 + (j & 1)));
          prog = true;
        }
        if (nS < nck && nS <= nYi + 1 && mbar_test(BAR(BAR_FULL0 + (nS & 1)), (nS >> 1) & 1) &&
            (nS < 2 || mbar_test(BAR(BAR_YFREE0 + (nS & 1)), ((nS >> 1) - 1) & 1))) {
          const int j = nS;
          tc_fence_after();
          TC_MARK(j, 10);
          issue_S(sb + (j & 1) * kStage, tmem + ((j & 1) ? TM_S1 : TM_S0));
          mma_commit(BAR(BAR_SREADY0 + (j & 1)));
          ++nS;
          if (stage_done(j)) mma_commit(BAR(BAR_EMPTY0 + (j & 1)));
          prog = true;
        }
        if (prog) {
          t_prog = globaltimer();
          nap = 32;
        } else {
          if (*abort_flag) {
            ok = false;
          } else if (globaltimer() - t_prog > lim) {
            *abort_flag = 1;
            if (a.err) atomicCAS(a.err, 0, (int)SSD_ERR_TIMEOUT);
            ok = false;
          } else {
            __nanosleep(nap);
            nap = nap < 256 ? 2 * nap : 256;
          }
        }
      }
      // no MMA may still be running when TMEM is released
      mma_commit(BAR(BAR_DONE));
      int never_abort = 0;
      mbar_wait(BAR(BAR_DONE), 0, &never_abort, a.err);
    }
  } else if (conv_index(warp) >= 0) {
    // ---------------------------------------------------------------- conv + SiLU -> X, w o X
    // Warp cw makes tokens 16cw..16cw+15; lane l channels 2l, 2l+1.  Raw row r of the w o X
    // buffer holds time t0-3+r; token s reads rows s..s+3 (a register window), then
    // overwrites row s with its w o X row and writes its X row to row s of X.  Rows
    // 16cw+16..+18 belong to the next warp's tokens, so every warp reads them before the
    // group barrier that precedes all writes.
    // SiLU(u) = u * sigmoid(u) = h + h * tanh(h) with h = u / 2.  The conv accumulates h
    // directly (halved weights) in fp16 pairs -- the precision of the MMA operand it feeds,
    // 11 significant bits -- and one half2 tanh serves both channels.  The last chunk of a
    // segment, whose newest tokens dominate the final state, uses fp32 and the exact SiLU.
    const int cw = conv_index(warp);
    const bool leader = (tid == 2 * 32);  // releases the stage
    const int ch = h * 64 + 2 * lane;
    const int W = kConv ? a.W : 0;
    float2 ew[4], bias2 = make_float2(0.f, 0.f);
#pragma unroll
    for (int j = 0; j < 4; ++j) {  // half the weight for the input at time t-3+j
      const int k = j - (4 - W);
      ew[j].x = (W > 0 && k >= 0) ? 0.5f * __bfloat162float(a.conv_w[(long long)ch * W + k]) : 0.f;
      ew[j].y = (W > 0 && k >= 0) ? 0.5f * __bfloat162float(a.conv_w[(long long)(ch + 1) * W + k]) : 0.f;
    }
    if (W > 0 && a.conv_b) {
      bias2.x = 0.5f * __bfloat162float(a.conv_b[ch]);
      bias2.y = 0.5f * __bfloat162float(a.conv_b[ch + 1]);
    }
    __half2 hw[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) hw[j] = __float22half2_rn(ew[j]);
    const __half2 hbias = __float22half2_rn(bias2);
    // byte offset of this lane's 4 bytes within a swizzled row r, by r mod 8
    uint32_t loff[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) loff[u] = ((uint32_t)((lane >> 2) ^ u) << 4) + ((uint32_t)(lane & 3) << 2);
    const int tok0 = kTokPerConvWarp * cw;  // multiple of 8
    for (int k = 0; k < nck; ++k) {
      const int st = k & 1, xb = k & 1, lb = (k + 1) & 1;
      const bool is_last = (k == last) && exact_last;
      // every thread waits for the chunk's inputs itself; one barrier per chunk (after the
      // boundary rows are read) keeps the warps together and makes an abort uniform, and each
      // warp signals its own rows of X and w o X (XREADY counts eight arrivals)
      bool ok = mbar_wait(BAR(BAR_FULLX0 + xb), (k >> 1) & 1, abort_flag, a.err, lim);
      if (ok) ok = mbar_wait(BAR(BAR_FULL0 + st), (k >> 1) & 1, abort_flag, a.err, lim);
      if (ok && k >= 2) ok = mbar_wait(BAR(BAR_XFREE0 + xb), ((k >> 1) - 1) & 1, abort_flag, a.err, lim);
      if (ok && is_last && k >= 1) ok = mbar_wait(BAR(BAR_XWFREE0 + lb), ((k - 1) >> 1) & 1, abort_flag, a.err, lim);
      if (leader) TC_MARK(k, 14);
      const float *cs = reinterpret_cast<const float *>(smem + st * kStage + OFF_CS);
      const float *dtv = reinterpret_cast<const float *>(smem + st * kStage + OFF_DT);
      const float cs_end = cs[QC - 1];
      const float wl = lane < kTokPerConvWarp ? __expf(cs_end - cs[tok0 + lane]) * dtv[tok0 + lane] : 0.f;
      const uint32_t wl2 = pack_f16(wl, wl);
      unsigned char *xt = smem + OFF_X + xb * kTile + tok0 * 128;   // row tok0
      unsigned char *xwt = smem + OFF_XW + xb * kXBuf + tok0 * 128;
      unsigned char *xlt = smem + OFF_XW + lb * kXBuf + tok0 * 128;
      // raw rows tok0 + r for r = 0..18 (tok0 is a multiple of 8, so row mod 8 = r mod 8)
#define RAW(r) (*reinterpret_cast<const uint32_t *>(xwt + (r) * 128 + loff[(r) & 7]))
      uint32_t r0 = RAW(0), r1 = RAW(1), r2 = RAW(2);
      const int t0 = t_begin + k * QC;
      if (cw == 0 && t0 == 0) {  // history before the first token comes from the conv cache
        uint32_t hist[3] = {0u, 0u, 0u};
#pragma unroll
        for (int j = 0; j < 3; ++j) {
          const int tau = j - 3;
          if (a.csi && W + tau >= 0)
            hist[j] = *reinterpret_cast<const uint32_t *>(a.csi + ((long long)b * W + (W + tau)) * a.conv_dim + ch);
        }
        r0 = hist[0];
        r1 = hist[1];
        r2 = hist[2];
      }
      const uint32_t nb0 = RAW(16), nb1 = RAW(17), nb2 = RAW(18);
      // all boundary rows read before any row is overwritten; a failed wait anywhere ends all
      if (named_bar_or(1, 256, !ok || *abort_flag != 0)) break;
      if (leader) {
        TC_MARK(k, 0);
        mbar_arrive(BAR(BAR_EMPTY0 + st));  // dt and prefix sums already read
      }
      // The token loop is compiled twice: the common chunks, and the last chunk of a segment.
      auto tokens = [&](auto last_tag) {
        constexpr bool kLast = decltype(last_tag)::value;
        if constexpr (!kLast) {
          __half2 xm3 = __float22half2_rn(unpack_bf16(r0)), xm2 = __float22half2_rn(unpack_bf16(r1)),
                  xm1 = __float22half2_rn(unpack_bf16(r2));
#pragma unroll 1
          for (int g = 0; g < 2; ++g) {
            __half2 xn[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const int nxt = 8 * g + u + 3;  // row of time t for token 8g+u
              uint32_t w3;
              if (nxt < 16) w3 = RAW(nxt);
              else w3 = nxt == 16 ? nb0 : (nxt == 17 ? nb1 : nb2);
              xn[u] = __float22half2_rn(unpack_bf16(w3));
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const int i = 8 * g + u;
              const __half2 x0 = xn[u];
              __half2 xo = x0;
              if (kConv) {
                __half2 acc = __hfma2(hw[0], xm3, hbias);
                acc = __hfma2(hw[1], xm2, acc);
                acc = __hfma2(hw[2], xm1, acc);
                acc = __hfma2(hw[3], x0, acc);
                xo = __hfma2(acc, h2tanh_approx(acc), acc);
              }
              const uint32_t off = i * 128 + loff[u];
              *reinterpret_cast<__half2 *>(xt + off) = xo;
              const uint32_t w2 = __shfl_sync(0xffffffffu, wl2, i);
              *reinterpret_cast<__half2 *>(xwt + off) = __hmul2(xo, *reinterpret_cast<const __half2 *>(&w2));
              xm3 = xm2;
              xm2 = xm1;
              xm1 = x0;
            }
          }
          return;
        }
        float2 xm3 = unpack_bf16(r0), xm2 = unpack_bf16(r1), xm1 = unpack_bf16(r2);
#pragma unroll 1
        for (int g = 0; g < 2; ++g) {
          float2 xn[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int nxt = 8 * g + u + 3;  // row of time t for token 8g+u
            uint32_t w3;
            if (nxt < 16) w3 = RAW(nxt);
            else w3 = nxt == 16 ? nb0 : (nxt == 17 ? nb1 : nb2);
            xn[u] = unpack_bf16(w3);
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int i = 8 * g + u;
            const float2 x0 = xn[u];
            float2 acc = x0;
            if (kConv) {
              acc = __ffma2_rn(ew[0], xm3, bias2);
              acc = __ffma2_rn(ew[1], xm2, acc);
              acc = __ffma2_rn(ew[2], xm1, acc);
              acc = __ffma2_rn(ew[3], x0, acc);
            }
            const uint32_t off = i * 128 + loff[u];
            {
              // The final state's chunk: its newest tokens dominate the final state, so X
              // comes from the fp32 SiLU and w o X is stored as the fp16 hi + lo parts of the
              // fp32 product.
              const float u0 = kConv ? silu(2.f * acc.x) : acc.x;
              const float u1 = kConv ? silu(2.f * acc.y) : acc.y;
              const float ws = __shfl_sync(0xffffffffu, wl, i);
              const float2 v = make_float2(u0 * ws, u1 * ws);
              const __half2 hi = __float22half2_rn(v);
              const float2 hf = __half22float2(hi);
              *reinterpret_cast<uint32_t *>(xt + off) = pack_f16(u0, u1);
              *reinterpret_cast<__half2 *>(xwt + off) = hi;
              *reinterpret_cast<uint32_t *>(xlt + off) = pack_f16(v.x - hf.x, v.y - hf.y);
            }
            xm3 = xm2;
            xm2 = xm1;
            xm1 = x0;
          }
        }
      };
      if (is_last) tokens(std::true_type{});
      else tokens(std::false_type{});
      if (leader) TC_MARK(k, 13);
#undef RAW
      fence_proxy_async();
      __syncwarp();
      if (leader) TC_MARK(k, 1);
      if (lane == 0) {
        mbar_arrive(BAR(BAR_XREADY0 + xb));
        if (is_last) mbar_arrive(BAR(BAR_XLOREADY));
      }
    }
  } else if (warp >= 10 && warp < 16) {
    // ---------------------------------------------------------------- S -> S~ (decay mask)
    // Row t of S sits in TMEM lane t, and a warp reaches only the 32 lanes of its SM
    // sub-partition (warp % 4): lane quarter q (rows 32q..32q+31) needs the blocks J <= q of
    // 32 columns, one to four of them.  Warps 12-15 own the quarters; warps 10 and 11 take
    // blocks 2..q of quarters 2 and 3, so that no warp handles more than two blocks.
    // S~ columns 32J..32J+31 go to the packed TMEM columns 16J..16J+15, which lie in S block
    // J/2: blocks 0 and 1 land in block 0, read by the same warp before; blocks 2 and 3 land
    // in block 1, so a helper stores only after its owner has read block 1 (named barrier
    // 4 or 5, owner arrives, helper waits).
    if (!kStateOnly) {
      const int q = warp & 3;
      const bool helper = warp < 12;
      const bool split = q >= 2;
      const int jlo = helper ? 2 : 0, jhi = (split && !helper) ? 1 : q;
      const int pair_bar = 4 + (q & 1);  // quarters 2 and 3
      const int t = 32 * q + lane;
      const bool leader = (tid == 14 * 32);
      float *cf = reinterpret_cast<float *>(smem + OFF_CF);
      const float Dh = a.D[h];
      for (int k = 0; k < nck; ++k) {
        const int st = k & 1;
        if (!wg_wait(BAR(BAR_FULL0 + st), (k >> 1) & 1, leader, 2, abort_flag, a.err, lim, 192)) break;
        if (!wg_wait(BAR(BAR_SREADY0 + st), (k >> 1) & 1, leader, 2, abort_flag, a.err, lim, 192)) break;
        tc_fence_after();
        float *cs = reinterpret_cast<float *>(smem + OFF_CSM);
        float *dtv = reinterpret_cast<float *>(smem + OFF_DTM);
        if (!helper) {  // private copies (the stage is released at once); column factor of
                        // column t: e^{r_J - cs_t} dt_t with r_J = cs at the end of t's block
          const float *scs = reinterpret_cast<const float *>(smem + st * kStage + OFF_CS);
          const float *sdt = reinterpret_cast<const float *>(smem + st * kStage + OFF_DT);
          const float rJ = scs[32 * (t >> 5) + 31];
          cs[t] = scs[t];
          dtv[t] = sdt[t];
          cf[t] = __expf(rJ - scs[t]) * sdt[t];
        }
        named_bar(2, 192);
        if (leader) mbar_arrive(BAR(BAR_EMPTY0 + st));
        if (leader) TC_MARK(k, 2);
        const float cst = cs[t];
        const uint32_t trow = tmem + (st ? TM_S1 : TM_S0) + ((uint32_t)(32 * q) << 16);
        // S~ = S * e^{cs_t - cs_s} dt_s, factored per block as rf_t * cf_s with rf_t = e^{cs_t -
        // r_J}; a block whose cs span is too steep to factor takes the direct exponential.  The
        // diagonal block J = q also applies the causal mask (column c <= row lane) and adds the
        // D x skip on its diagonal.
#pragma unroll 1
        for (int J = jlo; J <= jhi; ++J) {
          float v[32];
          tmem_ld32(trow + 32 * J, v);
          tmem_ld_wait();
          if (split && !helper && J == 1) {  // block 1 read: the helper may write over it
            tc_fence_before();
            named_bar_arrive(pair_bar, 64);
          }
          const float rJ = cs[32 * J + 31];
          if (cs[32 * J] - rJ > 60.f) {
#pragma unroll
            for (int c = 0; c < 32; ++c) v[c] *= __expf(fminf(cst - cs[32 * J + c], 0.f)) * dtv[32 * J + c];
          } else {
            const float rf = __expf(cst - rJ);
            const float2 rf2 = make_float2(rf, rf);
            const float4 *cf4 = reinterpret_cast<const float4 *>(cf + 32 * J);
#pragma unroll
            for (int qq = 0; qq < 8; ++qq) {
              const float4 c4 = cf4[qq];
              const float2 lo = __fmul2_rn(__fmul2_rn(make_float2(v[4 * qq], v[4 * qq + 1]), rf2),
                                           make_float2(c4.x, c4.y));
              const float2 hi = __fmul2_rn(__fmul2_rn(make_float2(v[4 * qq + 2], v[4 * qq + 3]), rf2),
                                           make_float2(c4.z, c4.w));
              v[4 * qq] = lo.x;
              v[4 * qq + 1] = lo.y;
              v[4 * qq + 2] = hi.x;
              v[4 * qq + 3] = hi.y;
            }
          }
          if (J == q) {
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              const float val = c <= lane ? v[c] : 0.f;
              v[c] = c == lane ? val + Dh : val;
            }
          }
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) pk[c] = pack_f16(v[2 * c], v[2 * c + 1]);
          if (helper && J == jlo) {  // the owner has read block 1
            named_bar(pair_bar, 64);
            tc_fence_after();
          }
          tmem_st16(trow + 16 * J, pk);
        }
        if (helper || !split) {  // blocks J > q lie above the diagonal: zeros
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) pk[c] = 0u;
#pragma unroll 1
          for (int J = q + 1; J < 4; ++J) tmem_st16(trow + 16 * J, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        named_bar(2, 192);
        if (leader) {
          TC_MARK(k, 3);
          mbar_arrive(BAR(BAR_STREADY0 + st));
        }
      }
    }
  } else if (warp >= 16) {
    // ---------------------------------------------------------------- state update + output
    const int ew = warp - 16;
    const int n = 32 * ew + lane;  // TMEM lane: state row n, output row t = n
    const bool leader = (tid == 19 * 32);
    const uint32_t lane_off = (uint32_t)(32 * ew) << 16;
    const long long bh = (long long)b * a.H + h;
    const long long hbase = seg * a.h_out_seg + bh * 8192;  // hout's offset in h_out
    float *hout = a.h_out ? a.h_out + hbase : nullptr;
    // tail mode: only the last segment writes, the state entering its last tail_chunks chunks
    const bool tail = a.tail_chunks > 0 && seg == (int)gridDim.x - 1 && hout != nullptr;
    const int tail_k = nck - 1 - a.tail_chunks;  // state after this chunk (-1: the initial state)
    {  // initial state -> TMEM (fp32) and the fp16 copy
      const float *hin = a.h_init ? a.h_init + seg * a.h_init_seg + bh * 8192 : nullptr;
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        float hr[32];
        uint32_t hu[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          hr[i] = hin ? hin[(32 * half + i) * 128 + n] : 0.f;
          hu[i] = __float_as_uint(hr[i]);
        }
        tmem_st32(tmem + TM_H + 32 * half + lane_off, hu);
        write_h_tile(smem, hr, n, half);
        if (tail && tail_k < 0) {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (in_bounds(hbase + (32 * half + i) * 128 + n, a.h_extent, a.err)) hout[(32 * half + i) * 128 + n] = hr[i];
        }
      }
      tmem_st_wait();
    }
    fence_proxy_async();
    tc_fence_before();
    named_bar(3, 128);
    if (leader) mbar_arrive(BAR(BAR_HREADY));
    float decay_sum = 0.f;
    for (int k = 0; k < nck; ++k) {
      const int st = k & 1;
      if (!wg_wait(BAR(BAR_FULL0 + st), (k >> 1) & 1, leader, 3, abort_flag, a.err, lim)) break;
      const float *cs = reinterpret_cast<const float *>(smem + st * kStage + OFF_CS);
      const float cs_end = cs[QC - 1];
      const float et = __expf(cs[n]);
      decay_sum += cs_end;
      const float ak = __expf(cs_end);
      named_bar(3, 128);  // every thread has read the prefix sums
      if (leader) mbar_arrive(BAR(BAR_EMPTY0 + st));
      // h_k = e^{cs_end} h_{k-1} + dH_k in TMEM, and its fp16 copy for MMA3 of chunk k+1, which
      // may overwrite the h tile once MMA3 of chunk k has read h_{k-1} from it
      const bool htile = !kStateOnly && k != last;
      if (leader) {
        bool ok = mbar_wait(BAR(BAR_DHREADY), k & 1, abort_flag, a.err, lim);
        if (ok && htile) mbar_wait(BAR(BAR_HTFREE), k & 1, abort_flag, a.err, lim);
      }
      if (named_bar_or(3, 128, *abort_flag != 0)) break;
      tc_fence_after();
      if (leader) TC_MARK(k, 4);
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        float dh[32], hr[32];
        tmem_ld32(tmem + TM_DH + 32 * half + lane_off, dh);
        tmem_ld32(tmem + TM_H + 32 * half + lane_off, hr);
        tmem_ld_wait();
        uint32_t hu[32];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float2 r = __ffma2_rn(make_float2(ak, ak), make_float2(hr[i], hr[i + 1]),
                                      make_float2(dh[i], dh[i + 1]));
          hr[i] = r.x;
          hr[i + 1] = r.y;
          hu[i] = __float_as_uint(r.x);
          hu[i + 1] = __float_as_uint(r.y);
        }
        tmem_st32(tmem + TM_H + 32 * half + lane_off, hu);
        if (htile) write_h_tile(smem, hr, n, half);
        if (tail && k == tail_k) {  // the state entering the tail, in fp32
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (in_bounds(hbase + (32 * half + i) * 128 + n, a.h_extent, a.err)) hout[(32 * half + i) * 128 + n] = hr[i];
        }
      }
      tmem_st_wait();
      if (htile) fence_proxy_async();
      tc_fence_before();
      named_bar(3, 128);
      if (leader) {
        mbar_arrive(BAR(BAR_DHFREE));  // dH read: MMA4 of chunk k+1 may overwrite it
        if (htile) {
          TC_MARK(k, 5);
          mbar_arrive(BAR(BAR_HREADY));
        }
      }
      if (!kStateOnly) {
        const int tok = t_begin + k * QC + n;
        const long long row = seq_base(a.cu, b, a.L) + tok;
        if (!wg_wait(BAR(BAR_YREADY0 + st), (k >> 1) & 1, leader, 3, abort_flag, a.err, lim)) break;
        tc_fence_after();
        if (leader) TC_MARK(k, 6);
        const uint32_t tYi = tmem + (st ? TM_S1 : TM_S0) + TM_YI_OFF + lane_off;
        const uint32_t tYs = tmem + (st ? TM_YS1 : TM_YS0) + lane_off;
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          float yi[32], ysv[32];
          tmem_ld32(tYi + 32 * half, yi);
          tmem_ld32(tYs + 32 * half, ysv);
          tmem_ld_wait();
          if (half == 1) {  // every product read: the buffers are free before the stores
            tc_fence_before();
            named_bar(3, 128);
            if (leader) {
              TC_MARK(k, 7);
              mbar_arrive(BAR(BAR_YFREE0 + st));
            }
          }
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float2 r = __ffma2_rn(make_float2(et, et), make_float2(ysv[i], ysv[i + 1]),
                                        make_float2(yi[i], yi[i + 1]));
            yi[i] = r.x;
            yi[i + 1] = r.y;
          }
          if (tok < t_end) {
            if (a.yh) {
              const long long yo = row * a.d_inner + h * 64 + 32 * half;
              uint4 *dst = reinterpret_cast<uint4 *>(a.yh + yo);
              if (in_bounds(yo + 31, a.y_extent, a.err)) {
#pragma unroll
                for (int i = 0; i < 4; ++i)
                  dst[i] = make_uint4(pack_f16(yi[8 * i], yi[8 * i + 1]), pack_f16(yi[8 * i + 2], yi[8 * i + 3]),
                                      pack_f16(yi[8 * i + 4], yi[8 * i + 5]), pack_f16(yi[8 * i + 6], yi[8 * i + 7]));
              }
            } else {
              const long long yo = row * a.ys + h * 64 + 32 * half;
              uint4 *dst = reinterpret_cast<uint4 *>(a.y + yo);
              if (in_bounds(yo + 31, a.y_extent, a.err)) {
#pragma unroll
                for (int i = 0; i < 4; ++i)
                  dst[i] = make_uint4(pack_bf16(yi[8 * i], yi[8 * i + 1]), pack_bf16(yi[8 * i + 2], yi[8 * i + 3]),
                                      pack_bf16(yi[8 * i + 4], yi[8 * i + 5]), pack_bf16(yi[8 * i + 6], yi[8 * i + 7]));
              }
            }
          }
        }
      }
    }
    if (*abort_flag == 0) {
      if (hout && a.tail_chunks == 0) {
        tc_fence_after();
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          float hr[32];
          tmem_ld32(tmem + TM_H + 32 * half + lane_off, hr);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (in_bounds(hbase + (32 * half + i) * 128 + n, a.h_extent, a.err)) hout[(32 * half + i) * 128 + n] = hr[i];
        }
      }
      if (a.seg_decay && n == 0) a.seg_decay[(long long)seg * a.B * a.H + bh] = __expf(decay_sum);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TM_COLS);
  }
#undef BAR
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  // resolved once (a function-local static is initialised exactly once, even under
  // concurrent first calls)
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
  }();
  return fn;
}

}  // namespace

bool tc_scan_available() {
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return false;
  return major == 10 && minor == 0 && encode_fn() != nullptr;
}

// mode 0: full scan of each segment from h_init (h0 or the inter-segment states) writing y;
// mode 1: state-only pass (zero initial state) writing per-segment states and decays.
cudaError_t launch_scan_tc(const PrefillPlan &p, int mode, cudaStream_t s) {
  auto enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap tm;
  const cuuint64_t C2 = 2ull * p.G * p.N;
  // a packed variable-length batch is one batch row of all its tokens
  const cuuint64_t T = p.cu ? (cuuint64_t)p.rows : (cuuint64_t)p.L, NB = p.cu ? 1 : (cuuint64_t)p.B;
  cuuint64_t dims[3] = {C2, T, NB};
  cuuint64_t strides[2] = {C2 * 2, C2 * 2 * T};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(&tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, p.bc, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  // raw x rows of one head: box of 64 channels x (128 + 3) tokens of the bf16 input
  CUtensorMap tmx;
  cuuint64_t xdims[3] = {(cuuint64_t)p.conv_dim, T, NB};
  cuuint64_t xstrides[2] = {(cuuint64_t)p.xs * 2, (cuuint64_t)p.xs * 2 * T};
  cuuint32_t xbox[3] = {64, kRawRows, 1};
  r = enc(&tmx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(p.xBC), xdims, xstrides, xbox,
          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  TcArgs a{};
  a.B = p.B; a.L = p.L; a.H = p.H; a.G = p.G; a.hpg = p.hpg; a.conv_dim = p.conv_dim;
  a.Lpad = p.Lpad; a.W = p.W; a.seg_len = p.seg_len;
  a.xBC = (const __nv_bfloat16 *)p.xBC; a.xs = p.xs; a.csi = (const __nv_bfloat16 *)p.csi;
  a.conv_w = (const __nv_bfloat16 *)p.conv_w; a.conv_b = (const __nv_bfloat16 *)p.conv_b;
  a.dte = p.dte_hm; a.cs = p.cs_hm; a.D = p.D;
  a.y = (__nv_bfloat16 *)p.y; a.ys = p.ys; a.err = p.err;
  if (p.norm_groups > 0 && !p.yh) return cudaErrorInvalidValue;  // the norm reads fp16 y
  a.yh = p.norm_groups > 0 ? p.yh : nullptr;
  a.wait_ns = p.stall_chunk1 > 0 ? p.stall_wait_ns : tc::kWaitLimitNs;
  a.debug_skip_chunk = p.stall_chunk1 - 1;
  a.d_inner = p.d_inner;
  a.cu = p.cu;
  a.y_extent = checked_extent(p, p.yh ? p.rows * p.d_inner : (p.rows - 1) * p.ys + p.d_inner);
  const long long seg_stride = (long long)p.B * p.H * p.P * p.N;
  dim3 grid(p.n_seg, p.H, p.B);
  cudaError_t e;
  if (mode == 1) {
    a.h_init = nullptr; a.h_init_seg = 0;
    a.h_out = p.seg_state; a.h_out_seg = seg_stride; a.seg_decay = p.seg_decay;
    a.h_extent = checked_extent(p, p.n_seg * seg_stride);
    auto kern = p.W > 0 ? ssd_scan_tc_kernel<true, true> : ssd_scan_tc_kernel<true, false>;
    e = set_smem_attr(kern, kSmemAlloc, s);
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreadsTC, kSmemAlloc, s>>>(tm, tmx, a);
  } else {
    if (p.n_seg > 1) {
      a.h_init = p.seg_state; a.h_init_seg = seg_stride;
    } else {
      a.h_init = p.h0; a.h_init_seg = 0;
    }
    // the last segment leaves the state before its last kTailChunks chunks; the fp32 tail pass
    // adds what those chunks contribute
    a.h_out = p.h_final; a.h_out_seg = 0; a.seg_decay = nullptr;
    a.h_extent = checked_extent(p, seg_stride);
    a.tail_chunks = p.tail_dh ? kTailChunks : 0;
    auto kern = p.W > 0 ? ssd_scan_tc_kernel<false, true> : ssd_scan_tc_kernel<false, false>;
    e = set_smem_attr(kern, kSmemAlloc, s);
    if (e != cudaSuccess) return e;
    // Programmatic dependent launch when the front end directly precedes the scan: the scan's
    // set-up (TMEM, barriers, tensor maps, its first raw x loads) overlaps the front end's tail,
    // and its producer waits for the front end before loading a stage.  Not after the
    // states-only pass (the state warps read its output at once).
    cudaLaunchConfig_t lc = {};
    lc.gridDim = grid; lc.blockDim = dim3(kThreadsTC); lc.dynamicSmemBytes = kSmemAlloc; lc.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = p.n_seg == 1 ? 1 : 0;
    lc.attrs = at; lc.numAttrs = 1;
    e = cudaLaunchKernelEx(&lc, kern, tm, tmx, a);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace ssd
