/*
 * ssd.h -- C ABI of libssd.so, a B200 (sm_100a) implementation of the Mamba-2
 * mixer's selective state-space scan ("SSD"), the data-parallel hot path of the
 * hybrid Mamba-Transformer described in "NVIDIA Nemotron Nano 2: An Accurate and
 * Efficient Hybrid Mamba-Transformer Reasoning Model".
 *
 * What the calls compute.  The layer hyper-parameters come from the Nemotron
 * Nano 2 pages (hyper.ai summary, section "Method"; neurohive.io article,
 * section "Model architecture"): 8 groups, state dimension N = 128, head
 * dimension P = 64, expansion 2, causal conv window W = 4, RMSNorm, no bias in
 * the linear layers; the SSM cache is float32 (neurohive.io article, section
 * "Deployment and usage").  The scan is the Mamba-2 scalar-decay recurrence,
 * per batch row b and head h (group g = h / (H/G)):
 *
 *   u      = SiLU(conv_b + causal depthwise conv1d_W(raw x|B|C channels))
 *   dt_t   = clamp(softplus(dt_raw_t + dt_bias_h), dt_min, dt_max)
 *   h_t    = exp(dt_t * A_h) * h_{t-1} + dt_t * x_t B_t^T        (P x N, fp32)
 *   y_t    = h_t C_t + D_h * x_t                                  (after the update)
 *   out_t  = (y_t * SiLU(z_t)) / sqrt(mean_group((y*SiLU(z))^2) + eps) * norm_w
 *
 * Layouts are row-major and token-major: a "row" is one token of one batch row,
 * channels contiguous, consecutive tokens `row_stride` elements apart, batch
 * rows `seqlen * row_stride` apart.  The raw conv input xBC holds, in order,
 * x (H*P channels, head h at h*P), B (G*N channels, group g at g*N) and C
 * (G*N channels).  conv_dim = H*P + 2*G*N, d_inner = H*P.
 *
 * Conventions for every call:
 *  - All pointers are DEVICE pointers owned by the caller.  The library never
 *    allocates device memory, frees or synchronises on these paths; it enqueues
 *    kernels on `stream` (a cudaStream_t, NULL = legacy default stream) and
 *    returns.  When the scan leaves SMs free, the tensor-core prefill runs its
 *    final-state pass (fp32 accuracy) on a library side stream, forked from
 *    `stream` after the front end and joined back into it within the same call,
 *    so every effect of the call is ordered on `stream` (stream capture
 *    included); otherwise the pass runs on `stream` after the scan.  That side
 *    stream and its two events are created by the first such call on each host
 *    thread and device and kept for the life of the process.
 *  - Argument errors are reported synchronously before anything is launched.
 *    Launch failures come back as SSD_ERR_CUDA.  Errors raised inside kernels
 *    (a bounded wait that gave up, or, in the debug build, an index check) are
 *    latched in a device word read by ssd_get_device_error().
 *  - Tensors read or written with 16-byte vectors (xBC, z, y, out, hidden, the
 *    weights, the conv caches, the states) must be 16-byte aligned, and their
 *    row strides must be multiples of 8 elements.
 *  - No C++ exception crosses this boundary.
 */
#ifndef SSD_H
#define SSD_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SSD_OK = 0,
  SSD_ERR_INVALID_ARG = 1,   /* missing/inconsistent argument or shape */
  SSD_ERR_UNSUPPORTED = 2,   /* valid request the library does not implement */
  SSD_ERR_ALIGNMENT = 3,     /* pointer or row stride not aligned as required */
  SSD_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed */
  SSD_ERR_TIMEOUT = 5,       /* a bounded device-side wait gave up */
  SSD_ERR_DEVICE_BOUNDS = 6, /* a device-side index check failed (checked builds) */
  SSD_ERR_WORKSPACE = 7      /* workspace missing, misaligned or too small */
} ssd_status_t;

typedef enum { SSD_F32 = 0, SSD_BF16 = 1 } ssd_dtype_t;

/* Kernel family selection (ssd_config_t.kernel). */
typedef enum {
  SSD_KERNEL_AUTO = 0,    /* tensor-core path for bf16 when supported, else SIMT */
  SSD_KERNEL_SIMT = 1,    /* fp32 CUDA-core chunked scan (any dtype) */
  SSD_KERNEL_TENSOR = 2   /* tcgen05/TMEM chunked scan (bf16 only; UNSUPPORTED otherwise) */
} ssd_kernel_t;

typedef struct {
  int batch;        /* B >= 1 */
  int seqlen;       /* L >= 0 tokens in this call (0: only the carries are copied) */
  int nheads;       /* H >= 1, multiple of ngroups */
  int headdim;      /* P; the library supports 64 */
  int dstate;       /* N; the library supports 128 */
  int ngroups;      /* G >= 1: B and C are shared by the H/G heads of a group */
  int chunk;        /* Q in {64, 128, 256}: tokens per chunk of the chunked scan */
  int conv_width;   /* W in 0..4; 0 = no conv and no activation (u = raw input) */
  int norm_groups;  /* 0 = no gate/norm (y is the output); else the z-gated RMSNorm over
                       groups of d_inner/norm_groups consecutive channels (z required) */
  float norm_eps;   /* RMSNorm epsilon (1e-5 in the workloads) */
  float dt_min;     /* clamp of the effective dt; 0 = no lower clamp */
  float dt_max;     /* upper clamp; +inf = none */
  int dt_softplus;  /* 1: dt = softplus(dt_raw + dt_bias); 0: dt = dt_raw + dt_bias */
  ssd_dtype_t io_dtype; /* dtype of xBC, dt, z, y, conv weights/caches, norm weight */
  int n_segments;   /* 0 = library choice; else split each sequence into this many segments
                       scanned in parallel and joined by the inter-segment state pass */
  ssd_kernel_t kernel;
  int norm_before_gate; /* 0: out = rmsnorm(y * silu(z)) * w (gate first, the default);
                           1: out = rmsnorm(y) * w * silu(z) (normalise first) */
} ssd_config_t;

typedef struct {
  const void *xBC;  long long xBC_row_stride;  /* [B, L, conv_dim] raw conv input */
  const void *dt;   long long dt_row_stride;   /* [B, L, H] raw dt (before dt_bias/softplus) */
  const void *z;    long long z_row_stride;    /* [B, L, d_inner] gate, or NULL if norm_groups == 0 */
  const float *A;       /* [H] decay rates (negative) */
  const float *D;       /* [H] skip weights */
  const float *dt_bias; /* [H] */
  const void *conv_w;   /* [conv_dim, W] (tap W-1 multiplies the newest input); NULL iff W == 0 */
  const void *conv_b;   /* [conv_dim] or NULL (= 0) */
  const void *norm_w;   /* [d_inner] or NULL (= 1) */
  const float *h0;      /* [B, H, P, N] initial state or NULL (= 0) */
  const void *conv_state_in; /* [B, W, conv_dim] last W raw inputs before this call, oldest
                                first; NULL = zeros */
  void *y;  long long y_row_stride;            /* [B, L, d_inner] output (io dtype) */
  float *h_final;       /* [B, H, P, N] state after the last token, or NULL; may alias h0 */
  void *conv_state_out; /* [B, W, conv_dim] or NULL: the last W raw inputs (bit-exact copies);
                           must not overlap conv_state_in */
  void *workspace;      /* device scratch of at least ssd_workspace_size() bytes, 256-B aligned */
  size_t workspace_bytes;
} ssd_prefill_args_t;

typedef struct {
  const void *xBC;  long long xBC_row_stride;  /* [B, conv_dim] new token's raw channels */
  const void *dt;   long long dt_row_stride;   /* [B, H] raw dt */
  const void *z;    long long z_row_stride;    /* [B, d_inner] or NULL if norm_groups == 0 */
  const float *A, *D, *dt_bias;                /* [H] */
  const void *conv_w, *conv_b, *norm_w;        /* as in ssd_prefill_args_t */
  float *state;               /* [B, H, P, N] fp32 SSM state, updated in place */
  const void *conv_state_in;  /* [B, W, conv_dim] cache before this token (required if W > 0) */
  void *conv_state_out;       /* [B, W, conv_dim] cache after it; must not overlap conv_state_in */
  void *y;  long long y_row_stride;            /* [B, d_inner] output */
} ssd_decode_args_t;

typedef struct {
  ssd_config_t ssd;   /* scan shape; io_dtype must be SSD_BF16; seqlen >= 1 */
  int d_model;        /* hidden width (multiple of 64) */
  float rms_eps;      /* input RMSNorm epsilon */
} ssd_mixer_config_t;

typedef struct {
  const void *hidden;  /* [B, L, d_model] bf16 */
  const void *rms_w;   /* [d_model] bf16 input-norm weight, or NULL (= 1) */
  const void *W_in;    /* [proj, d_model] bf16, proj = 2*d_inner + 2*G*N + H; output columns
                          are ordered z | x | B | C | dt */
  const void *W_out;   /* [d_model, d_inner] bf16 */
  const float *A, *D, *dt_bias;                /* [H] */
  const void *conv_w, *conv_b, *norm_w;        /* bf16, as in ssd_prefill_args_t */
  const float *h0; const void *conv_state_in;  /* optional carries in */
  float *h_final;  void *conv_state_out;       /* optional carries out */
  void *out;           /* [B, L, d_model] bf16 */
  void *workspace;     /* at least ssd_mixer_workspace_size() bytes, 256-B aligned */
  size_t workspace_bytes;
} ssd_mixer_args_t;

/* Bytes of scratch ssd_prefill needs for this configuration (0 if the config is invalid). */
size_t ssd_workspace_size(const ssd_config_t *cfg);

/* Chunked prefill over seqlen tokens with optional state/conv-cache carry in and out.
 * Computes y (or the gated, normalised output when norm_groups > 0), the final SSM state
 * and the conv cache.  Splitting a sequence into consecutive calls, each fed the previous
 * call's h_final and conv_state_out, gives the same result as one call (up to rounding). */
ssd_status_t ssd_prefill(const ssd_config_t *cfg, const ssd_prefill_args_t *args, void *stream);

/* Variable-length batch: nseq sequences packed back to back along the token axis, each with
 * its own initial state and conv cache (the state is reset at every sequence boundary).
 *  cu_seqlens: HOST array of nseq + 1 non-decreasing offsets, cu_seqlens[0] = 0; sequence i
 *    is packed tokens [cu_seqlens[i], cu_seqlens[i+1]) (an empty sequence copies its carries).
 *  cfg: batch = 1 and seqlen = cu_seqlens[nseq] (all tokens); the token tensors of args
 *    (xBC, dt, z, y) are the packed [seqlen, ...] rows; h0 / h_final are [nseq, H, P, N] and
 *    conv_state_in / conv_state_out [nseq, W, conv_dim] (NULL as in ssd_prefill; with
 *    h_final NULL the pass that computes the final states' last chunks is skipped).
 *  workspace: at least ssd_varlen_workspace_size(cfg, cu_seqlens, nseq) bytes.
 * On the tensor-core path (bf16 with the shapes its fused front end takes) the whole packed
 * batch is one pass on `stream`, one launch of each kernel, bit-exact against one
 * ssd_prefill per sequence; other paths run the prefill of each sequence in turn.  Returns the
 * first error (argument errors, including inconsistent offsets, as SSD_ERR_INVALID_ARG). */
size_t ssd_varlen_workspace_size(const ssd_config_t *cfg, const int *cu_seqlens, int nseq);
ssd_status_t ssd_prefill_varlen(const ssd_config_t *cfg, const ssd_prefill_args_t *args,
                                const int *cu_seqlens, int nseq, void *stream);

/* Sequence parallelism (one exchange).  A sequence too long for one GPU is split into spans
 * of consecutive tokens, one per rank.  The recurrence is linear in the state, so the state
 * entering span k is h_in[k] = lambda_{k-1} h_in[k-1] + s_{k-1} (h_in[0] = h0), where s_k is
 * the state span k produces from a zero state and lambda_k = exp(sum over its tokens of
 * dt A), per (batch row, head).  This is the chunked form's inter-chunk recurrence of the
 * Mamba-2 scan applied at span granularity; the pages fix only the fp32 state it carries
 * (neurohive.io article, section "Deployment and usage") and 128k-token contexts (abstract).
 * Per rank: (1) ssd_prefill_span_state on its span; (2) the caller all-gathers (s_k,
 * lambda_k) over the ranks (its own collective, e.g. NCCL all-gather: n_spans * B*H*P*N +
 * n_spans * B*H floats); (3) ssd_span_prefix gives h_in[k]; (4) ssd_prefill on the span with
 * h0 = h_in[own k] gives its y, and the last rank's h_final is the sequence's final state.
 * The conv of a span's first W-1 tokens reads the previous span's last W raw rows: each rank
 * is given them as conv_state_in (a W-row halo of its input), so no exchange is needed for it.
 *
 * ssd_prefill_span_state: args as for ssd_prefill (xBC, dt, A, dt_bias, conv_w, conv_b,
 *   conv_state_in and the workspace are used; y, D, z, norm_w, h0, h_final and
 *   conv_state_out are ignored and may be NULL).  Writes span_state [B, H, P, N] fp32
 *   (16-byte aligned) and span_decay [B, H] fp32.  seqlen = 0 gives zeros and ones.  Errors
 *   as for ssd_prefill. */
ssd_status_t ssd_prefill_span_state(const ssd_config_t *cfg, const ssd_prefill_args_t *args,
                                    float *span_state, float *span_decay, void *stream);

/* ssd_span_prefix: span_states [n_spans, B, H, P, N] and span_decays [n_spans, B, H] (fp32,
 * span-major, as an all-gather leaves them); h0 [B, H, P, N] or NULL (zero).  Writes
 * h_in [n_spans, B, H, P, N] (the state entering each span; may be span_states itself, in
 * place; otherwise the two must not overlap) and/or h_final [B, H, P, N] (the state after the
 * last span); either may be NULL but not both.  Device pointers, 16-byte aligned
 * (SSD_ERR_ALIGNMENT); headdim * dstate a multiple of 4 (SSD_ERR_INVALID_ARG). */
ssd_status_t ssd_span_prefix(const float *span_states, const float *span_decays, int n_spans,
                             int batch, int nheads, int headdim, int dstate, const float *h0,
                             float *h_in, float *h_final, void *stream);

/* One token per batch row: conv-cache shift + conv + SiLU, softplus dt, the state update
 * h = exp(dt A) h + dt x B^T (fp32 state in place), y = h C + D x, optional gated RMSNorm.
 * cfg->seqlen and cfg->chunk are ignored.  norm_groups must be 0 or a multiple of ngroups. */
ssd_status_t ssd_decode_step(const ssd_config_t *cfg, const ssd_decode_args_t *args, void *stream);

/* Bytes of scratch mamba2_mixer_forward needs. */
size_t ssd_mixer_workspace_size(const ssd_mixer_config_t *cfg);

/* Full Mamba-2 mixer layer: input RMSNorm -> in_proj (no bias) -> conv/SiLU + chunked scan +
 * z-gated RMSNorm -> out_proj (no bias).  The residual add belongs to the caller. */
ssd_status_t mamba2_mixer_forward(const ssd_mixer_config_t *cfg, const ssd_mixer_args_t *args,
                                  void *stream);

/* Human-readable name of a status code (static storage). */
const char *ssd_status_string(ssd_status_t status);

/* Size of the fixed device scratch that ssd_prefill_noalloc uses (64 MiB per device). */
#define SSD_NOALLOC_WORKSPACE_BYTES (64ull << 20)

/* ssd_prefill for callers that must not allocate device memory themselves (their device memory
 * belongs to a framework allocator or a fixed pool, or they cannot afford the device-wide
 * synchronisation a cudaMalloc may cause).  Inputs and outputs are passed exactly as for
 * ssd_prefill; args->workspace and args->workspace_bytes are ignored.  Scratch comes from one
 * array of SSD_NOALLOC_WORKSPACE_BYTES that the library reserves on every device it is loaded
 * on and keeps until the process exits; the call itself allocates and frees nothing.
 *  - Returns SSD_ERR_WORKSPACE when ssd_workspace_size(cfg) exceeds that size.  On the
 *    tensor-core path that is about 2,900 tokens per call of a 128-head, 8-group layer with
 *    the gated norm, and about 12,000 without it; more for smaller layers.
 *  - The first call on a device looks up the array's device address; make that first call
 *    before starting any stream capture.
 *  - All calls share the array: calls whose kernels may run at the same time (different
 *    streams without ordering, several host threads) race and must be ordered by the caller.
 *    Nothing needs clearing between calls.
 * This entry point is a property of this library; the paper has no counterpart to it. */
ssd_status_t ssd_prefill_noalloc(const ssd_config_t *cfg, const ssd_prefill_args_t *args, void *stream);

/* Waits for `stream`, then returns and clears the status latched by kernels on this device
 * (SSD_OK, SSD_ERR_TIMEOUT or SSD_ERR_DEVICE_BOUNDS). */
ssd_status_t ssd_get_device_error(void *stream);

/* Version of this library as MAJOR*10000 + MINOR*100 + PATCH. */
int ssd_version(void);

/* Test hook for the failure path of the bounded device waits (not for production use).
 * While set (chunk >= 0), every tensor-core prefill scan withholds the loads of that chunk's
 * B/C tile, so the CTAs that wait for it give up after wait_limit_ns nanoseconds of device
 * time instead of the normal 2 s, leave cleanly (loads drained, MMAs complete, tensor memory
 * released) and latch SSD_ERR_TIMEOUT for ssd_get_device_error().  The outputs of such a call
 * are undefined.  chunk < 0 turns the hook off.  Process-wide; not thread-safe with respect
 * to prefills running concurrently on other host threads. */
void ssd_test_stall_scan(int chunk, unsigned long long wait_limit_ns);

/* Debug build with device-side index checks (libssd_debug.so, compiled with
 * -DSSD_DEBUG_BOUNDS): the kernels check the index of each store to y, the final and segment
 * states, the tail pass's buffers, the fused front end's B/C and dt buffers and the gated
 * norm's output against the buffer's extent.  An index outside it latches
 * SSD_ERR_DEVICE_BOUNDS for ssd_get_device_error() and the store is skipped; nothing traps.
 * Returns 1 in that build, 0 in the normal one (where the checks compile away). */
int ssd_debug_bounds_build(void);

/* Test hook of the debug build: the index checks allow 1/denom of each buffer's extent
 * (denom <= 1 restores the full extents), so that a call with valid buffers trips them while
 * every access stays inside its allocation.  Process-wide; no effect in the normal build. */
void ssd_test_bounds_scale(int denom);

/* Kernel tracing for measurement tools.  While enabled, every kernel the library launches
 * is bracketed by two CUDA events recorded on the stream it is launched on (so the timing
 * covers exactly that kernel).  Off by default; do not enable it while a stream is being
 * captured into a CUDA graph. */
typedef struct {
  char name[48];  /* kernel family, e.g. "ssd_scan_simt" */
  float ms;       /* device time between the two events */
} ssd_trace_record_t;

/* Turns tracing on (on != 0) or off; returns the previous setting. */
int ssd_trace_enable(int on);

/* Waits for the recorded events, copies up to max_records records (oldest first) into out,
 * discards all records and returns the number copied (-1 on a CUDA error). */
int ssd_trace_read(ssd_trace_record_t *out, int max_records);

#ifdef __cplusplus
}
#endif

#endif /* SSD_H */
