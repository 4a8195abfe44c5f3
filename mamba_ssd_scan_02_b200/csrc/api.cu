// api.cu -- the C ABI of libssd.so: argument validation, workspace layout and the launch
// sequence of each entry point.  Nothing here allocates device memory or synchronises on the
// compute paths.
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "plan.h"

namespace ssd {

// The device error word that kernels latch failures into (one per device).
__device__ int g_device_error_word;

namespace {

// Test hook (ssd_test_stall_scan): chunk index + 1 whose stage the tensor-core scan withholds,
// and the wait limit its bounded waits then use; 0 = off.
std::atomic<int> g_stall_chunk1{0};
std::atomic<unsigned long long> g_stall_wait_ns{0};
// Test hook (ssd_test_bounds_scale): the debug build's index checks allow 1/denom of each
// buffer's extent; 1 = off.
std::atomic<int> g_bounds_denom{1};

constexpr int kMaxDevices = 64;
constexpr long long kTargetCtas = 2 * 148;  // scan CTAs wanted in flight (2 per B200 SM)
constexpr size_t kAlign = 256;

int *device_error_ptr() {
  static std::mutex mu;
  static int *ptrs[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (!ptrs[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error_word) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<int *>(p);
  }
  return ptrs[dev];
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
size_t elt_size(ssd_dtype_t t) { return t == SSD_F32 ? 4 : 2; }

bool ranges_overlap(const void *a, size_t na, const void *b, size_t nb) {
  const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
  return pa < pb + nb && pb < pa + na;
}

ssd_status_t check_config(const ssd_config_t *c, bool prefill) {
  if (!c) return SSD_ERR_INVALID_ARG;
  if (c->batch < 1 || c->nheads < 1 || c->ngroups < 1 || c->seqlen < 0) return SSD_ERR_INVALID_ARG;
  if (c->nheads % c->ngroups != 0) return SSD_ERR_INVALID_ARG;
  if (c->io_dtype != SSD_F32 && c->io_dtype != SSD_BF16) return SSD_ERR_INVALID_ARG;
  if (c->headdim != kHeadDim || c->dstate != kDState) return SSD_ERR_UNSUPPORTED;
  if (prefill && c->chunk != 64 && c->chunk != 128 && c->chunk != 256) return SSD_ERR_UNSUPPORTED;
  if (c->conv_width < 0 || c->conv_width > 4) return SSD_ERR_UNSUPPORTED;
  const long long d_inner = (long long)c->nheads * c->headdim;
  if (c->norm_groups < 0 || (c->norm_groups > 0 && d_inner % c->norm_groups != 0))
    return SSD_ERR_INVALID_ARG;
  if (!(c->norm_eps >= 0.f) || !(c->dt_min <= c->dt_max) || isnan(c->dt_min)) return SSD_ERR_INVALID_ARG;
  if (c->n_segments < 0) return SSD_ERR_INVALID_ARG;
  if (c->norm_before_gate != 0 && c->norm_before_gate != 1) return SSD_ERR_INVALID_ARG;
  if (c->kernel != SSD_KERNEL_AUTO && c->kernel != SSD_KERNEL_SIMT && c->kernel != SSD_KERNEL_TENSOR)
    return SSD_ERR_INVALID_ARG;
  if (c->batch > 65535 || c->nheads > 65535 || c->seqlen > (1 << 21))
    return SSD_ERR_UNSUPPORTED;  // grid limits
  return SSD_OK;
}

// Internal sequence segments: each a whole number of `tile`-token chunks, enough
// (b, h, segment) CTAs to fill `target` CTA slots, and at least four tiles long.
void choose_segments(const ssd_config_t *c, int tile, long long target, int *n_seg, int *seg_len) {
  const int L = c->seqlen;
  int n = c->n_segments;
  if (n == 0) {
    const long long bh = (long long)c->batch * c->nheads;
    n = 1;
    if (bh < target && L > 4 * tile) {
      n = (int)(target / bh);
      n = n < L / (4 * tile) ? n : L / (4 * tile);
      if (n > 64) n = 64;
      if (n < 1) n = 1;
    }
  }
  if (n < 1) n = 1;
  long long len = L > 0 ? ((long long)L + n - 1) / n : tile;
  len = (len + tile - 1) / tile * tile;
  *seg_len = (int)len;
  *n_seg = L > 0 ? (int)((L + len - 1) / len) : 1;
}

constexpr int kTcTile = 128;       // tokens per chunk of the tensor-core scan
constexpr long long kTcTarget = 148;  // one tensor-core scan CTA per SM

void simt_segments(const ssd_config_t *c, int *n, int *len) {
  choose_segments(c, c->chunk, kTargetCtas, n, len);
}
void tc_segments(const ssd_config_t *c, int *n, int *len) {
  choose_segments(c, kTcTile, kTcTarget, n, len);
}

// The scan path a prefill with this config takes on the current device: the tensor-core scan
// for bf16 unless the CUDA-core one is requested (an explicit tensor-core request on a device
// without it is refused later, but is sized for that path).
bool prefill_uses_tc(const ssd_config_t *c) {
  if (c->kernel == SSD_KERNEL_SIMT) return false;
  if (c->kernel == SSD_KERNEL_TENSOR) return true;
  return c->io_dtype == SSD_BF16 && tc_scan_available();
}

// On the tensor path the scan hands y to the gated norm in fp16 (2 bytes per channel): the
// norm's pass reads it with z once, so the scan's output stage needs no memory read.
bool tc_norm_f16(const ssd_config_t *c) { return c->io_dtype == SSD_BF16 && c->norm_groups > 0; }

// The two scan paths use the workspace differently; the layouts overlap (a call uses one),
// and the size asked for is that of the path the call takes.
struct WsLayout {
  // CUDA-core path
  size_t u, dte, yf, seg_state, seg_decay, simt_end;
  // tensor-core path
  size_t tc_bc, tc_dte, tc_cs, tc_yf, tc_yh, tc_seg_state, tc_seg_decay, tc_dh, tc_end;
  int Lpad;
  size_t total;
};

WsLayout prefill_layout(const ssd_config_t *c) {
  WsLayout w{};
  const size_t T = (size_t)c->batch * c->seqlen;
  const size_t d_inner = (size_t)c->nheads * c->headdim;
  const size_t conv_dim = d_inner + 2 * (size_t)c->ngroups * c->dstate;
  const size_t state = (size_t)c->batch * c->nheads * c->headdim * c->dstate * 4;
  int n_seg, seg_len;
  simt_segments(c, &n_seg, &seg_len);
  size_t off = 0;
  w.u = off;    off = round_up(off + T * conv_dim * 4, kAlign);
  w.dte = off;  off = round_up(off + T * c->nheads * 4, kAlign);
  w.yf = off;   if (c->norm_groups > 0) off = round_up(off + T * d_inner * 4, kAlign);
  w.seg_state = w.seg_decay = off;
  if (n_seg > 1) {
    off = round_up(off + (size_t)n_seg * state, kAlign);
    w.seg_decay = off;
    off = round_up(off + (size_t)n_seg * c->batch * c->nheads * 4, kAlign);
  }
  w.simt_end = off;
  tc_segments(c, &n_seg, &seg_len);
  w.Lpad = (int)((c->seqlen + kTcTile - 1) / kTcTile * kTcTile);
  off = 0;
  w.tc_bc = off;   off = round_up(off + T * 2 * c->ngroups * c->dstate * 2, kAlign);
  w.tc_dte = off;  off = round_up(off + (size_t)c->batch * c->nheads * w.Lpad * 4, kAlign);
  w.tc_cs = off;   off = round_up(off + (size_t)c->batch * c->nheads * w.Lpad * 4, kAlign);
  w.tc_yf = w.tc_yh = off;
  if (tc_norm_f16(c)) {
    off = round_up(off + T * d_inner * 2, kAlign);
  } else if (c->norm_groups > 0) {
    off = round_up(off + T * d_inner * 4, kAlign);
  }
  w.tc_seg_state = w.tc_seg_decay = off;
  if (n_seg > 1) {
    off = round_up(off + (size_t)n_seg * state, kAlign);
    w.tc_seg_decay = off;
    off = round_up(off + (size_t)n_seg * c->batch * c->nheads * 4, kAlign);
  }
  w.tc_dh = off;   off = round_up(off + state + (size_t)c->batch * c->nheads * 4, kAlign);
  w.tc_end = off;
  w.total = prefill_uses_tc(c) ? w.tc_end : w.simt_end;
  return w;
}

ssd_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA; }

#define SSD_TRY(expr)                            \
  do {                                           \
    cudaError_t e_ = (expr);                     \
    if (e_ != cudaSuccess) return SSD_ERR_CUDA;  \
  } while (0)

// Per host thread and device: a side stream and two events that run the tail pass beside the
// output scan (made on first use and kept for the life of the process).  Per thread, so
// that a fork is always joined before the same objects are recorded again.
struct SideStream {
  cudaStream_t s;
  cudaEvent_t fork, join;
};
cudaError_t side_stream(SideStream **out) {
  thread_local SideStream tls[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  SideStream &ss = tls[dev];
  if (!ss.s) {
    SideStream n{};
    if ((e = cudaStreamCreateWithFlags(&n.s, cudaStreamNonBlocking)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&n.fork, cudaEventDisableTiming)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&n.join, cudaEventDisableTiming)) != cudaSuccess) {
      if (n.fork) cudaEventDestroy(n.fork);
      cudaStreamDestroy(n.s);
      return e;
    }
    ss = n;
  }
  *out = &ss;
  return cudaSuccess;
}

// Once the side stream has been forked from the caller's stream, joins it back on every exit
// (an early error return included): the caller's stream, or a graph being captured from it,
// never ends the call with work of this call still outstanding on the side stream.
struct SideJoin {
  SideStream *side = nullptr;
  cudaStream_t s = nullptr;
  bool forked = false;
  cudaError_t join() {
    if (!forked) return cudaSuccess;
    forked = false;
    cudaError_t e = cudaEventRecord(side->join, side->s);
    if (e != cudaSuccess) return e;
    return cudaStreamWaitEvent(s, side->join, 0);
  }
  ~SideJoin() { join(); }
};

// Span mode (sequence parallelism): instead of y and the final state, the call leaves the
// state its tokens produce from a zero state, and their total decay exp(sum dt A), per
// (batch row, head).  y, h0, z and the norm, and the outgoing conv cache are not used.
struct SpanOut {
  float *state;  // [B, H, P, N]
  float *decay;  // [B, H]
};

// Variable-length batch in one pass (tensor path): nseq sequences packed back to back, with
// host offsets cu_host[0..nseq]; the plan is that of a batch of nseq rows of the longest
// length, whose row b reads and writes the packed rows of sequence b (PrefillPlan::cu).
struct VarlenIn {
  const int *cu_host;
  int nseq, Lmax;
  long long total;
};

// Workspace of the one-pass variable-length prefill: the plan's layout, then the device copy
// of the offsets.
size_t varlen_cu_offset(const ssd_config_t *cv) { return round_up(prefill_layout(cv).total, kAlign); }

ssd_status_t run_prefill(const ssd_config_t *c_in, const ssd_prefill_args_t *a, cudaStream_t s,
                         const SpanOut *span = nullptr, const VarlenIn *vl = nullptr) {
  ssd_config_t c_span;
  const ssd_config_t *c = c_in;
  if (span && c_in) {  // the norm does not touch the state
    c_span = *c_in;
    c_span.norm_groups = 0;
    c = &c_span;
  }
  if (vl && c_in) {  // nseq rows of the longest length, one internal segment per sequence
    c_span = *c_in;
    c_span.batch = vl->nseq;
    c_span.seqlen = vl->Lmax;
    c_span.n_segments = 1;
    c = &c_span;
  }
  ssd_status_t st = check_config(c, true);
  if (st != SSD_OK) return st;
  if (!a) return SSD_ERR_INVALID_ARG;
  if (span && (!span->state || !span->decay || !aligned16(span->state))) return SSD_ERR_INVALID_ARG;
  const int H = c->nheads, P = c->headdim, N = c->dstate, G = c->ngroups, W = c->conv_width;
  const long long d_inner = (long long)H * P, conv_dim = d_inner + 2LL * G * N;
  const size_t es = elt_size(c->io_dtype);
  const long long rows = vl ? vl->total : (long long)c->batch * c->seqlen;  // token rows
  const bool has_tokens = rows > 0;
  if (has_tokens) {
    if (!a->xBC || !a->dt || !a->A || !a->dt_bias || (!span && (!a->D || !a->y))) return SSD_ERR_INVALID_ARG;
    if (W > 0 && !a->conv_w) return SSD_ERR_INVALID_ARG;
    if (c->norm_groups > 0 && !a->z) return SSD_ERR_INVALID_ARG;
    if (a->xBC_row_stride < conv_dim || a->dt_row_stride < H || (!span && a->y_row_stride < d_inner))
      return SSD_ERR_INVALID_ARG;
    if (c->norm_groups > 0 && a->z_row_stride < d_inner) return SSD_ERR_INVALID_ARG;
    if (!aligned16(a->xBC) || a->xBC_row_stride % 8) return SSD_ERR_ALIGNMENT;
    if (!span && (!aligned16(a->y) || (a->z && !aligned16(a->z)) || a->y_row_stride % 8 ||
                  (a->z && a->z_row_stride % 8)))
      return SSD_ERR_ALIGNMENT;
  }
  if ((a->h0 && !aligned16(a->h0)) || (a->h_final && !aligned16(a->h_final)) ||
      (a->conv_state_in && !aligned16(a->conv_state_in)) ||
      (a->conv_state_out && !aligned16(a->conv_state_out)))
    return SSD_ERR_ALIGNMENT;
  const size_t cache_bytes = (size_t)c->batch * W * conv_dim * es;
  if (a->conv_state_in && a->conv_state_out &&
      ranges_overlap(a->conv_state_in, cache_bytes, a->conv_state_out, cache_bytes))
    return SSD_ERR_INVALID_ARG;

  PrefillPlan p{};
  p.B = c->batch; p.L = c->seqlen; p.H = H; p.P = P; p.N = N; p.G = G; p.Q = c->chunk; p.W = W;
  p.norm_groups = c->norm_groups; p.hpg = H / G; p.d_inner = (int)d_inner; p.conv_dim = (int)conv_dim;
  p.nbg = c->norm_before_gate;
  p.eps = c->norm_eps; p.dt_min = c->dt_min; p.dt_max = c->dt_max; p.softplus = c->dt_softplus;
  p.bf16 = c->io_dtype == SSD_BF16;
  p.xBC = a->xBC; p.xs = a->xBC_row_stride; p.dt = a->dt; p.ds = a->dt_row_stride;
  p.z = a->z; p.zs = a->z_row_stride; p.A = a->A; p.D = a->D; p.dt_bias = a->dt_bias;
  p.conv_w = a->conv_w; p.conv_b = a->conv_b; p.norm_w = a->norm_w; p.h0 = a->h0;
  p.csi = a->conv_state_in; p.y = a->y; p.ys = a->y_row_stride; p.h_final = a->h_final;
  p.cso = a->conv_state_out;
  if (span) {
    p.z = nullptr; p.norm_w = nullptr; p.h0 = nullptr; p.y = nullptr; p.h_final = nullptr;
    p.cso = nullptr;
  }
  p.err = device_error_ptr();
  p.rows = rows;
  p.stall_chunk1 = g_stall_chunk1.load();
  p.stall_wait_ns = g_stall_wait_ns.load();
  p.bounds_denom = g_bounds_denom.load();

  if (span) {
    // the combine of internal segments (or of none) into the span's own state and decay
    auto combine = [&](const char *name) {
      return traced(name, s, [&] {
        return launch_span_prefix(p.seg_state, nullptr, p.seg_decay, p.n_seg, (long long)p.B * p.H,
                                  p.P * p.N, nullptr, span->state, span->decay, s);
      });
    };
    if (!has_tokens) {
      p.n_seg = 0;
      return from_cuda(combine("ssd_span_combine"));
    }
  }
  if (!has_tokens) return from_cuda(traced("ssd_carry", s, [&] { return launch_carry_only(p, s); }));

  const bool use_tc = prefill_uses_tc(c);
  if (use_tc && (!p.bf16 || !tc_scan_available())) return SSD_ERR_UNSUPPORTED;
  if (vl && (!use_tc || !front_tc_fusable(p))) return SSD_ERR_UNSUPPORTED;
  const WsLayout lay = prefill_layout(c);
  const size_t ws_need = vl ? varlen_cu_offset(c) + (size_t)(vl->nseq + 1) * sizeof(int) : lay.total;
  if (a->workspace_bytes < ws_need || (ws_need && !a->workspace) ||
      (reinterpret_cast<uintptr_t>(a->workspace) % kAlign) != 0)
    return SSD_ERR_WORKSPACE;
  char *ws = static_cast<char *>(a->workspace);
  if (vl) {  // the offsets on the device (a pageable host source is staged before the return)
    int *cu_dev = reinterpret_cast<int *>(ws + varlen_cu_offset(c));
    SSD_TRY(cudaMemcpyAsync(cu_dev, vl->cu_host, (size_t)(vl->nseq + 1) * sizeof(int),
                            cudaMemcpyHostToDevice, s));
    p.cu = cu_dev;
  }

  if (use_tc) {
    tc_segments(c, &p.n_seg, &p.seg_len);
    p.Lpad = lay.Lpad;
    p.bc = ws + lay.tc_bc;
    p.dte_hm = reinterpret_cast<float *>(ws + lay.tc_dte);
    p.cs_hm = reinterpret_cast<float *>(ws + lay.tc_cs);
    const bool norm_f16 = tc_norm_f16(c);
    p.yf = c->norm_groups > 0 && !norm_f16 ? reinterpret_cast<float *>(ws + lay.tc_yf) : nullptr;
    p.yh = norm_f16 ? reinterpret_cast<__half *>(ws + lay.tc_yh) : nullptr;
    p.seg_state = p.n_seg > 1 ? reinterpret_cast<float *>(ws + lay.tc_seg_state) : nullptr;
    p.seg_decay = p.n_seg > 1 ? reinterpret_cast<float *>(ws + lay.tc_seg_decay) : nullptr;
    p.tail_dh = p.h_final ? reinterpret_cast<float *>(ws + lay.tc_dh) : nullptr;
    p.tail_dec = p.h_final ? p.tail_dh + (size_t)c->batch * c->nheads * c->headdim * c->dstate : nullptr;
    // The outgoing conv cache may be written before the scan unless it overlaps an input
    // that later kernels read.
    const size_t x_span = ((size_t)rows - 1) * (size_t)a->xBC_row_stride * es + (size_t)conv_dim * es;
    const size_t z_span = a->z ? ((size_t)rows - 1) * (size_t)a->z_row_stride * es + (size_t)d_inner * es : 0;
    const bool fused = front_tc_fusable(p);
    const bool cso_early = fused && !(a->conv_state_out && (ranges_overlap(a->conv_state_out, cache_bytes, a->xBC, x_span) ||
                                                            (a->z && ranges_overlap(a->conv_state_out, cache_bytes, a->z, z_span))));
    if (fused) {
      SSD_TRY(traced("ssd_front", s, [&] { return launch_front_tc(p, cso_early, s); }));
    } else {
      SSD_TRY(traced("ssd_dt_cumsum", s, [&] { return launch_dt_cumsum(p, p.dte_hm, p.cs_hm, p.Lpad, s); }));
      SSD_TRY(traced("ssd_bc_conv", s, [&] { return launch_bc_conv_f16(p, s); }));
    }
    if (span) {
      if (p.n_seg == 1) {
        p.seg_state = span->state;
        p.seg_decay = span->decay;
        return from_cuda(traced("ssd_scan_tc_states", s, [&] { return launch_scan_tc(p, 1, s); }));
      }
      SSD_TRY(traced("ssd_scan_tc_states", s, [&] { return launch_scan_tc(p, 1, s); }));
      return from_cuda(traced("ssd_span_combine", s, [&] {
        return launch_span_prefix(p.seg_state, nullptr, p.seg_decay, p.n_seg, (long long)p.B * p.H,
                                  p.P * p.N, nullptr, span->state, span->decay, s);
      }));
    }
    // The tail pass needs only the front end's outputs.  When the scan leaves enough SMs free
    // it is forked onto a side stream right after the front end and launched after the scan,
    // so that it takes those SMs, and joined before the fold; otherwise it runs after the scan
    // on this stream and folds into h_final itself.
    SideJoin side;
    const bool tail_beside = p.tail_dh && tail_beside_scan(p);
    if (tail_beside) {
      SSD_TRY(side_stream(&side.side));
      side.s = s;
      SSD_TRY(cudaEventRecord(side.side->fork, s));
      SSD_TRY(cudaStreamWaitEvent(side.side->s, side.side->fork, 0));
      side.forked = true;
    }
    if (p.n_seg > 1) {
      SSD_TRY(traced("ssd_scan_tc_states", s, [&] { return launch_scan_tc(p, 1, s); }));
      SSD_TRY(traced("ssd_state_pass", s, [&] { return launch_state_pass(p, s); }));
    }
    SSD_TRY(traced("ssd_scan_tc", s, [&] { return launch_scan_tc(p, 0, s); }));
    if (side.forked) {
      SSD_TRY(traced("ssd_state_tail", side.side->s, [&] { return launch_state_tail(p, false, side.side->s); }));
      SSD_TRY(side.join());
      SSD_TRY(traced("ssd_tail_fold", s, [&] { return launch_tail_fold(p, s); }));
    } else if (p.tail_dh) {  // no room beside the scan: after it, folding into h_final itself
      SSD_TRY(traced("ssd_state_tail", s, [&] { return launch_state_tail(p, true, s); }));
    }
    if (p.norm_groups > 0) {
      SSD_TRY(traced("ssd_gated_norm", s, [&] { return launch_gated_norm(p, s); }));
    }
    if (!cso_early) SSD_TRY(traced("ssd_conv_state_out", s, [&] { return launch_conv_state_out(p, s); }));
    return SSD_OK;
  }

  simt_segments(c, &p.n_seg, &p.seg_len);
  p.u = reinterpret_cast<float *>(ws + lay.u);
  p.dte = reinterpret_cast<float *>(ws + lay.dte);
  p.yf = c->norm_groups > 0 ? reinterpret_cast<float *>(ws + lay.yf) : nullptr;
  p.seg_state = p.n_seg > 1 ? reinterpret_cast<float *>(ws + lay.seg_state) : nullptr;
  p.seg_decay = p.n_seg > 1 ? reinterpret_cast<float *>(ws + lay.seg_decay) : nullptr;
  SSD_TRY(traced("ssd_dt", s, [&] { return launch_dt(p, s); }));
  SSD_TRY(traced("ssd_conv_silu", s, [&] { return launch_conv_silu_f32(p, s); }));
  if (span) {
    if (p.n_seg == 1) {
      p.seg_state = span->state;
      p.seg_decay = span->decay;
      return from_cuda(traced("ssd_scan_simt_states", s, [&] { return launch_scan_simt(p, 1, s); }));
    }
    SSD_TRY(traced("ssd_scan_simt_states", s, [&] { return launch_scan_simt(p, 1, s); }));
    return from_cuda(traced("ssd_span_combine", s, [&] {
      return launch_span_prefix(p.seg_state, nullptr, p.seg_decay, p.n_seg, (long long)p.B * p.H,
                                p.P * p.N, nullptr, span->state, span->decay, s);
    }));
  }
  if (p.n_seg == 1) {
    SSD_TRY(traced("ssd_scan_simt", s, [&] { return launch_scan_simt(p, 0, s); }));
  } else {
    SSD_TRY(traced("ssd_scan_simt_states", s, [&] { return launch_scan_simt(p, 1, s); }));
    SSD_TRY(traced("ssd_state_pass", s, [&] { return launch_state_pass(p, s); }));
    SSD_TRY(traced("ssd_scan_simt", s, [&] { return launch_scan_simt(p, 2, s); }));
  }
  if (p.norm_groups > 0) SSD_TRY(traced("ssd_gated_norm", s, [&] { return launch_gated_norm(p, s); }));
  SSD_TRY(traced("ssd_conv_state_out", s, [&] { return launch_conv_state_out(p, s); }));
  return SSD_OK;
}

ssd_status_t run_decode(const ssd_config_t *c, const ssd_decode_args_t *a, cudaStream_t s) {
  ssd_status_t st = check_config(c, false);
  if (st != SSD_OK) return st;
  if (!a) return SSD_ERR_INVALID_ARG;
  const int H = c->nheads, P = c->headdim, N = c->dstate, G = c->ngroups, W = c->conv_width;
  const long long d_inner = (long long)H * P, conv_dim = d_inner + 2LL * G * N;
  if (!a->xBC || !a->dt || !a->A || !a->D || !a->dt_bias || !a->y || !a->state)
    return SSD_ERR_INVALID_ARG;
  if (W > 0 && (!a->conv_w || !a->conv_state_in || !a->conv_state_out)) return SSD_ERR_INVALID_ARG;
  if (c->norm_groups > 0 && (!a->z || c->norm_groups % G != 0)) {
    return !a->z ? SSD_ERR_INVALID_ARG : SSD_ERR_UNSUPPORTED;
  }
  if (a->xBC_row_stride < conv_dim || a->dt_row_stride < H || a->y_row_stride < d_inner ||
      (c->norm_groups > 0 && a->z_row_stride < d_inner))
    return SSD_ERR_INVALID_ARG;
  if (!aligned16(a->xBC) || !aligned16(a->y) || !aligned16(a->state) || (a->z && !aligned16(a->z)) ||
      (a->conv_state_in && !aligned16(a->conv_state_in)) ||
      (a->conv_state_out && !aligned16(a->conv_state_out)) || a->xBC_row_stride % 8 ||
      a->y_row_stride % 8 || (a->z && a->z_row_stride % 8))
    return SSD_ERR_ALIGNMENT;
  const size_t cache_bytes = (size_t)c->batch * W * conv_dim * elt_size(c->io_dtype);
  if (W > 0 && ranges_overlap(a->conv_state_in, cache_bytes, a->conv_state_out, cache_bytes))
    return SSD_ERR_INVALID_ARG;
  if ((long long)(H / G) * P > 8192) return SSD_ERR_UNSUPPORTED;  // group staged in shared memory
  DecodePlan p{};
  p.B = c->batch; p.H = H; p.P = P; p.N = N; p.G = G; p.W = W; p.norm_groups = c->norm_groups;
  p.hpg = H / G; p.d_inner = (int)d_inner; p.conv_dim = (int)conv_dim; p.eps = c->norm_eps;
  p.nbg = c->norm_before_gate;
  p.dt_min = c->dt_min; p.dt_max = c->dt_max; p.softplus = c->dt_softplus;
  p.bf16 = c->io_dtype == SSD_BF16;
  p.xBC = a->xBC; p.xs = a->xBC_row_stride; p.dt = a->dt; p.ds = a->dt_row_stride; p.z = a->z;
  p.zs = a->z_row_stride; p.A = a->A; p.D = a->D; p.dt_bias = a->dt_bias; p.conv_w = a->conv_w;
  p.conv_b = a->conv_b; p.norm_w = a->norm_w; p.state = a->state; p.csi = a->conv_state_in;
  p.cso = a->conv_state_out; p.y = a->y; p.ys = a->y_row_stride;
  return from_cuda(traced("ssd_decode", s, [&] { return launch_decode(p, s); }));
}

// The input RMSNorm is folded into the in_proj GEMM: rmsnorm(x) W_in^T = diag(r) x (W_in diag(w))^T,
// with r the per-row factor (computed by a light pass over x) applied in the GEMM's epilogue and
// the norm weight w folded into a copy of W_in, so the normalised activations never reach HBM.
struct MixerLayout {
  size_t rs, wf, zxbcdt, g, ssd, total;
  ssd_config_t scfg;
};

MixerLayout mixer_layout(const ssd_mixer_config_t *m) {
  MixerLayout l{};
  l.scfg = m->ssd;
  const size_t T = (size_t)m->ssd.batch * m->ssd.seqlen;
  const size_t d_inner = (size_t)m->ssd.nheads * m->ssd.headdim;
  const size_t proj = 2 * d_inner + 2 * (size_t)m->ssd.ngroups * m->ssd.dstate + m->ssd.nheads;
  const size_t proj_pad = round_up(proj, 8);
  size_t off = 0;
  l.rs = off;      off = round_up(off + T * 4, kAlign);
  l.wf = off;      off = round_up(off + proj * m->d_model * 2, kAlign);
  l.zxbcdt = off;  off = round_up(off + T * proj_pad * 2, kAlign);
  l.g = off;       off = round_up(off + T * d_inner * 2, kAlign);
  l.ssd = off;     off = round_up(off + prefill_layout(&l.scfg).total, kAlign);
  l.total = off;
  return l;
}

ssd_status_t run_mixer(const ssd_mixer_config_t *m, const ssd_mixer_args_t *a, cudaStream_t s) {
  if (!m || !a) return SSD_ERR_INVALID_ARG;
  ssd_status_t st = check_config(&m->ssd, true);
  if (st != SSD_OK) return st;
  if (m->ssd.io_dtype != SSD_BF16 || m->ssd.seqlen < 1) return SSD_ERR_UNSUPPORTED;
  if (m->d_model < 64 || m->d_model % 64 != 0) return SSD_ERR_UNSUPPORTED;
  if (!a->hidden || !a->W_in || !a->W_out || !a->out) return SSD_ERR_INVALID_ARG;
  if (!aligned16(a->hidden) || !aligned16(a->W_in) || !aligned16(a->W_out) || !aligned16(a->out) ||
      (a->rms_w && !aligned16(a->rms_w)))
    return SSD_ERR_ALIGNMENT;
  const MixerLayout l = mixer_layout(m);
  if (!a->workspace || a->workspace_bytes < l.total ||
      (reinterpret_cast<uintptr_t>(a->workspace) % kAlign) != 0)
    return SSD_ERR_WORKSPACE;
  const int H = m->ssd.nheads, P = m->ssd.headdim, N = m->ssd.dstate, G = m->ssd.ngroups;
  const long long d_inner = (long long)H * P, conv_dim = d_inner + 2LL * G * N;
  const long long proj = 2 * d_inner + 2LL * G * N + H, proj_pad = (long long)round_up(proj, 8);
  const long long T = (long long)m->ssd.batch * m->ssd.seqlen;
  if (T > INT32_MAX) return SSD_ERR_UNSUPPORTED;
  char *ws = static_cast<char *>(a->workspace);
  float *rs = reinterpret_cast<float *>(ws + l.rs);
  void *zx = ws + l.zxbcdt, *g = ws + l.g;
  const void *w_in = a->W_in;
  SSD_TRY(traced("ssd_rms_rowscale", s, [&] {
    return launch_rms_rowscale_bf16(a->hidden, rs, T, m->d_model, m->rms_eps, s);
  }));
  if (a->rms_w) {
    SSD_TRY(traced("ssd_fold_rms_w", s, [&] {
      return launch_fold_cols_bf16(a->W_in, a->rms_w, ws + l.wf, proj, m->d_model, s);
    }));
    w_in = ws + l.wf;
  }
  SSD_TRY(traced("gemm_in_proj", s, [&] {
    return launch_gemm_bf16_tn(a->hidden, m->d_model, w_in, m->d_model, zx, proj_pad, (int)T, (int)proj,
                               m->d_model, s, rs);
  }));
  const __nv_bfloat16 *zxb = static_cast<const __nv_bfloat16 *>(zx);
  ssd_prefill_args_t pa{};
  pa.z = zxb;                         pa.z_row_stride = proj_pad;
  pa.xBC = zxb + d_inner;             pa.xBC_row_stride = proj_pad;
  pa.dt = zxb + d_inner + conv_dim;   pa.dt_row_stride = proj_pad;
  pa.A = a->A; pa.D = a->D; pa.dt_bias = a->dt_bias; pa.conv_w = a->conv_w; pa.conv_b = a->conv_b;
  pa.norm_w = a->norm_w; pa.h0 = a->h0; pa.conv_state_in = a->conv_state_in;
  pa.y = g; pa.y_row_stride = d_inner; pa.h_final = a->h_final; pa.conv_state_out = a->conv_state_out;
  pa.workspace = ws + l.ssd; pa.workspace_bytes = l.total - l.ssd;
  st = run_prefill(&l.scfg, &pa, s);
  if (st != SSD_OK) return st;
  SSD_TRY(traced("gemm_out_proj", s, [&] {
    return launch_gemm_bf16_tn(g, d_inner, a->W_out, d_inner, a->out, m->d_model, (int)T, m->d_model,
                               (int)d_inner, s);
  }));
  return SSD_OK;
}

}  // namespace

// Tensor-core GEMM on sm_100 when the operands satisfy TMA's alignment rules, else CUDA cores.
cudaError_t launch_gemm_bf16_tn(const void *A, long long lda, const void *Bm, long long ldb, void *C,
                                long long ldc, int M, int N, int K, cudaStream_t s, const float *row_scale) {
  const bool aligned = aligned16(A) && aligned16(Bm) && aligned16(C) && lda % 8 == 0 && ldb % 8 == 0 &&
                       ldc % 8 == 0;
  if (aligned && tc_scan_available())
    return launch_gemm_tc_bf16_tn(A, lda, Bm, ldb, C, ldc, M, N, K, device_error_ptr(), s, row_scale);
  return launch_gemm_simt_bf16_tn(A, lda, Bm, ldb, C, ldc, M, N, K, s, row_scale);
}

}  // namespace ssd

using namespace ssd;

extern "C" {

size_t ssd_workspace_size(const ssd_config_t *cfg) {
  if (check_config(cfg, true) != SSD_OK) return 0;
  return prefill_layout(cfg).total;
}

ssd_status_t ssd_prefill(const ssd_config_t *cfg, const ssd_prefill_args_t *args, void *stream) {
  return run_prefill(cfg, args, static_cast<cudaStream_t>(stream));
}

ssd_status_t ssd_decode_step(const ssd_config_t *cfg, const ssd_decode_args_t *args, void *stream) {
  return run_decode(cfg, args, static_cast<cudaStream_t>(stream));
}

// Variable-length batch.  On the tensor path (bf16, shapes the fused front end takes) it is one
// pass: the front end, the scan (a CTA per (sequence, head)), the tail pass and the norm each
// launch once for all the packed sequences.  Otherwise each packed sequence is one batch-1
// prefill on the same stream, its token tensors addressed at the sequence's first row and its
// carries at its index.
static VarlenIn varlen_in(const int *cu, int nseq) {
  VarlenIn v{cu, nseq, 0, cu[nseq]};
  for (int i = 0; i < nseq; ++i) v.Lmax = std::max(v.Lmax, cu[i + 1] - cu[i]);
  return v;
}

static bool varlen_ok(const ssd_config_t *cfg, const int *cu, int nseq) {
  if (!cfg || !cu || nseq < 1 || cfg->batch != 1 || cu[0] != 0 || cu[nseq] != cfg->seqlen) return false;
  for (int i = 0; i < nseq; ++i)
    if (cu[i + 1] < cu[i]) return false;
  return true;
}

size_t ssd_varlen_workspace_size(const ssd_config_t *cfg, const int *cu_seqlens, int nseq) {
  if (!varlen_ok(cfg, cu_seqlens, nseq) || check_config(cfg, true) != SSD_OK) return 0;
  size_t ws = 0;
  if (prefill_uses_tc(cfg)) {  // the one-pass layout (the call may still take the loop)
    const VarlenIn v = varlen_in(cu_seqlens, nseq);
    ssd_config_t cv = *cfg;
    cv.batch = nseq; cv.seqlen = v.Lmax; cv.n_segments = 1;
    ws = varlen_cu_offset(&cv) + (size_t)(nseq + 1) * sizeof(int);
  }
  for (int i = 0; i < nseq; ++i) {
    ssd_config_t c = *cfg;
    c.seqlen = cu_seqlens[i + 1] - cu_seqlens[i];
    const size_t w = prefill_layout(&c).total;
    ws = w > ws ? w : ws;
  }
  return ws;
}

ssd_status_t ssd_prefill_varlen(const ssd_config_t *cfg, const ssd_prefill_args_t *args,
                                const int *cu_seqlens, int nseq, void *stream) {
  if (!args || !varlen_ok(cfg, cu_seqlens, nseq)) return SSD_ERR_INVALID_ARG;
  ssd_status_t st = check_config(cfg, true);
  if (st != SSD_OK) return st;
  const size_t es = cfg->io_dtype == SSD_F32 ? 4 : 2;
  const long long d_inner = (long long)cfg->nheads * cfg->headdim;
  const long long conv_dim = d_inner + 2LL * cfg->ngroups * cfg->dstate;
  const long long state = (long long)cfg->nheads * cfg->headdim * cfg->dstate;
  const long long cache = (long long)cfg->conv_width * conv_dim;
  if (prefill_uses_tc(cfg)) {
    const VarlenIn v = varlen_in(cu_seqlens, nseq);
    st = run_prefill(cfg, args, static_cast<cudaStream_t>(stream), nullptr, &v);
    if (st != SSD_ERR_UNSUPPORTED) return st;
  }
  for (int i = 0; i < nseq; ++i) {
    ssd_config_t c = *cfg;
    const long long t0 = cu_seqlens[i];
    c.seqlen = cu_seqlens[i + 1] - cu_seqlens[i];
    ssd_prefill_args_t a = *args;
    auto at = [](const void *p, long long bytes) -> const char * {
      return p ? static_cast<const char *>(p) + bytes : nullptr;
    };
    a.xBC = at(args->xBC, t0 * args->xBC_row_stride * es);
    a.dt = at(args->dt, t0 * args->dt_row_stride * es);
    a.z = at(args->z, t0 * args->z_row_stride * es);
    a.y = const_cast<char *>(at(args->y, t0 * args->y_row_stride * es));
    a.h0 = reinterpret_cast<const float *>(at(args->h0, i * state * 4));
    a.h_final = reinterpret_cast<float *>(const_cast<char *>(at(args->h_final, i * state * 4)));
    a.conv_state_in = at(args->conv_state_in, i * cache * es);
    a.conv_state_out = const_cast<char *>(at(args->conv_state_out, i * cache * es));
    st = run_prefill(&c, &a, static_cast<cudaStream_t>(stream));
    if (st != SSD_OK) return st;
  }
  return SSD_OK;
}

size_t ssd_mixer_workspace_size(const ssd_mixer_config_t *cfg) {
  if (!cfg || check_config(&cfg->ssd, true) != SSD_OK) return 0;
  return mixer_layout(cfg).total;
}

ssd_status_t mamba2_mixer_forward(const ssd_mixer_config_t *cfg, const ssd_mixer_args_t *args,
                                  void *stream) {
  return run_mixer(cfg, args, static_cast<cudaStream_t>(stream));
}

const char *ssd_status_string(ssd_status_t s) {
  switch (s) {
    case SSD_OK: return "SSD_OK";
    case SSD_ERR_INVALID_ARG: return "SSD_ERR_INVALID_ARG: missing or inconsistent argument";
    case SSD_ERR_UNSUPPORTED: return "SSD_ERR_UNSUPPORTED: shape or option not implemented";
    case SSD_ERR_ALIGNMENT: return "SSD_ERR_ALIGNMENT: pointer or row stride not 16-byte aligned";
    case SSD_ERR_CUDA: return "SSD_ERR_CUDA: CUDA runtime call or launch failed";
    case SSD_ERR_TIMEOUT: return "SSD_ERR_TIMEOUT: a bounded device-side wait gave up";
    case SSD_ERR_DEVICE_BOUNDS: return "SSD_ERR_DEVICE_BOUNDS: device-side index check failed";
    case SSD_ERR_WORKSPACE: return "SSD_ERR_WORKSPACE: workspace missing, misaligned or too small";
  }
  return "unknown ssd_status_t";
}

ssd_status_t ssd_get_device_error(void *stream) {
  int *p = device_error_ptr();
  if (!p) return SSD_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int v = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return SSD_ERR_CUDA;
  if (cudaMemcpy(&v, p, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return SSD_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpy(p, &zero, sizeof zero, cudaMemcpyHostToDevice) != cudaSuccess) return SSD_ERR_CUDA;
  }
  return static_cast<ssd_status_t>(v);
}

ssd_status_t ssd_prefill_span_state(const ssd_config_t *cfg, const ssd_prefill_args_t *args,
                                    float *span_state, float *span_decay, void *stream) {
  const SpanOut out{span_state, span_decay};
  return run_prefill(cfg, args, static_cast<cudaStream_t>(stream), &out);
}

ssd_status_t ssd_span_prefix(const float *span_states, const float *span_decays, int n_spans,
                             int batch, int nheads, int headdim, int dstate, const float *h0,
                             float *h_in, float *h_final, void *stream) {
  if (n_spans < 0 || batch < 0 || nheads < 0 || headdim < 1 || dstate < 1 ||
      (headdim * dstate) % 4 != 0)
    return SSD_ERR_INVALID_ARG;
  if (n_spans > 0 && (!span_states || !span_decays)) return SSD_ERR_INVALID_ARG;
  if (!h_in && !h_final) return SSD_ERR_INVALID_ARG;
  if ((span_states && !aligned16(span_states)) || (h0 && !aligned16(h0)) ||
      (h_in && !aligned16(h_in)) || (h_final && !aligned16(h_final)))
    return SSD_ERR_ALIGNMENT;
  const long long BH = (long long)batch * nheads;
  if (h_in && h_in != span_states && n_spans > 0) {
    const size_t bytes = (size_t)n_spans * BH * headdim * dstate * sizeof(float);
    if (ranges_overlap(h_in, bytes, span_states, bytes)) return SSD_ERR_INVALID_ARG;
  }
  return from_cuda(traced("ssd_span_prefix", static_cast<cudaStream_t>(stream), [&] {
    return launch_span_prefix(span_states, h_in, span_decays, n_spans, BH, headdim * dstate, h0,
                              h_final, nullptr, static_cast<cudaStream_t>(stream));
  }));
}

int ssd_version(void) { return 100; }

void ssd_test_stall_scan(int chunk, unsigned long long wait_limit_ns) {
  g_stall_wait_ns.store(wait_limit_ns);
  g_stall_chunk1.store(chunk >= 0 ? chunk + 1 : 0);
}

int ssd_debug_bounds_build(void) {
#ifdef SSD_DEBUG_BOUNDS
  return 1;
#else
  return 0;
#endif
}

void ssd_test_bounds_scale(int denom) { g_bounds_denom.store(denom > 1 ? denom : 1); }

}  // extern "C"
