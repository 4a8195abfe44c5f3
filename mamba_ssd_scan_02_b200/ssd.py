"""Thin Python binding of libssd.so (include/ssd.h): argument marshalling only.

Every computation runs in the CUDA library.  PyTorch supplies device memory and the
current stream; this module builds the C structs, allocates outputs/workspace with
torch when the caller does not pass them, and turns status codes into exceptions.
There is no CPU fallback: if libssd.so cannot be loaded, ``load()`` raises.

Tensor conventions (all on one CUDA device, channels contiguous):
  xBC [B, L, conv_dim] (row stride may exceed conv_dim), dt [B, L, H], z [B, L, d_inner],
  A, D, dt_bias [H] float32, conv_w [conv_dim, W], conv_b [conv_dim], norm_w [d_inner],
  h0 / h_final [B, H, 64, 128] float32, conv caches [B, W, conv_dim], y [B, L, d_inner].
bf16 io uses torch.bfloat16; the fp32 io path uses torch.float32.
"""
from __future__ import annotations

import ctypes
import math
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libssd.so")
# the same library with device-side index checks (-DSSD_DEBUG_BOUNDS), for tests
DEBUG_LIB_PATH = os.path.join(_HERE, "libssd_debug.so")

SSD_F32, SSD_BF16 = 0, 1
KERNEL_AUTO, KERNEL_SIMT, KERNEL_TENSOR = 0, 1, 2
STATUS = {0: "SSD_OK", 1: "SSD_ERR_INVALID_ARG", 2: "SSD_ERR_UNSUPPORTED", 3: "SSD_ERR_ALIGNMENT",
          4: "SSD_ERR_CUDA", 5: "SSD_ERR_TIMEOUT", 6: "SSD_ERR_DEVICE_BOUNDS", 7: "SSD_ERR_WORKSPACE"}

c_int, c_float, c_ll, vp, c_size = (ctypes.c_int, ctypes.c_float, ctypes.c_longlong, ctypes.c_void_p,
                                    ctypes.c_size_t)


class SsdError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


class SsdConfig(ctypes.Structure):
    _fields_ = [("batch", c_int), ("seqlen", c_int), ("nheads", c_int), ("headdim", c_int),
                ("dstate", c_int), ("ngroups", c_int), ("chunk", c_int), ("conv_width", c_int),
                ("norm_groups", c_int), ("norm_eps", c_float), ("dt_min", c_float),
                ("dt_max", c_float), ("dt_softplus", c_int), ("io_dtype", c_int),
                ("n_segments", c_int), ("kernel", c_int), ("norm_before_gate", c_int)]


class PrefillArgs(ctypes.Structure):
    _fields_ = [("xBC", vp), ("xBC_row_stride", c_ll), ("dt", vp), ("dt_row_stride", c_ll),
                ("z", vp), ("z_row_stride", c_ll), ("A", vp), ("D", vp), ("dt_bias", vp),
                ("conv_w", vp), ("conv_b", vp), ("norm_w", vp), ("h0", vp), ("conv_state_in", vp),
                ("y", vp), ("y_row_stride", c_ll), ("h_final", vp), ("conv_state_out", vp),
                ("workspace", vp), ("workspace_bytes", c_size)]


class DecodeArgs(ctypes.Structure):
    _fields_ = [("xBC", vp), ("xBC_row_stride", c_ll), ("dt", vp), ("dt_row_stride", c_ll),
                ("z", vp), ("z_row_stride", c_ll), ("A", vp), ("D", vp), ("dt_bias", vp),
                ("conv_w", vp), ("conv_b", vp), ("norm_w", vp), ("state", vp),
                ("conv_state_in", vp), ("conv_state_out", vp), ("y", vp), ("y_row_stride", c_ll)]


class MixerConfig(ctypes.Structure):
    _fields_ = [("ssd", SsdConfig), ("d_model", c_int), ("rms_eps", c_float)]


class MixerArgs(ctypes.Structure):
    _fields_ = [("hidden", vp), ("rms_w", vp), ("W_in", vp), ("W_out", vp), ("A", vp), ("D", vp),
                ("dt_bias", vp), ("conv_w", vp), ("conv_b", vp), ("norm_w", vp), ("h0", vp),
                ("conv_state_in", vp), ("h_final", vp), ("conv_state_out", vp), ("out", vp),
                ("workspace", vp), ("workspace_bytes", c_size)]


class TraceRecord(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 48), ("ms", c_float)]


EXPORTS = ("ssd_workspace_size", "ssd_prefill", "ssd_decode_step", "ssd_mixer_workspace_size",
           "mamba2_mixer_forward", "ssd_status_string", "ssd_get_device_error", "ssd_version",
           "ssd_trace_enable", "ssd_trace_read", "ssd_prefill_noalloc", "ssd_varlen_workspace_size",
           "ssd_prefill_varlen", "ssd_test_stall_scan", "ssd_prefill_span_state", "ssd_span_prefix",
           "ssd_debug_bounds_build", "ssd_test_bounds_scale")

def debug_bounds_build() -> bool:
    """True for the library built with device-side index checks (libssd_debug.so)."""
    return bool(load().ssd_debug_bounds_build())


def test_bounds_scale(denom: int) -> None:
    """Test hook of the debug build: its index checks allow 1/denom of each buffer's extent
    (1 restores them), so a call with valid buffers trips them without any access leaving its
    allocation."""
    load().ssd_test_bounds_scale(int(denom))


NOALLOC_WORKSPACE_BYTES = 64 << 20

_lib = None


def load(path: str = LIB_PATH):
    """Load libssd.so (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libssd.so not built ({path}); run python -m mamba_ssd_scan_02_b200.build")
    try:  # let torch load its CUDA runtime first so the process has a single runtime
        import torch  # noqa: F401
    except ImportError:
        pass
    lib = ctypes.CDLL(path)
    lib.ssd_workspace_size.restype = c_size
    lib.ssd_workspace_size.argtypes = [ctypes.POINTER(SsdConfig)]
    lib.ssd_prefill.restype = c_int
    lib.ssd_prefill.argtypes = [ctypes.POINTER(SsdConfig), ctypes.POINTER(PrefillArgs), vp]
    lib.ssd_decode_step.restype = c_int
    lib.ssd_decode_step.argtypes = [ctypes.POINTER(SsdConfig), ctypes.POINTER(DecodeArgs), vp]
    lib.ssd_mixer_workspace_size.restype = c_size
    lib.ssd_mixer_workspace_size.argtypes = [ctypes.POINTER(MixerConfig)]
    lib.mamba2_mixer_forward.restype = c_int
    lib.mamba2_mixer_forward.argtypes = [ctypes.POINTER(MixerConfig), ctypes.POINTER(MixerArgs), vp]
    lib.ssd_status_string.restype = ctypes.c_char_p
    lib.ssd_status_string.argtypes = [c_int]
    lib.ssd_get_device_error.restype = c_int
    lib.ssd_get_device_error.argtypes = [vp]
    lib.ssd_version.restype = c_int
    lib.ssd_version.argtypes = []
    lib.ssd_varlen_workspace_size.restype = ctypes.c_size_t
    lib.ssd_varlen_workspace_size.argtypes = [ctypes.POINTER(SsdConfig), ctypes.POINTER(c_int), c_int]
    lib.ssd_prefill_varlen.restype = c_int
    lib.ssd_prefill_varlen.argtypes = [ctypes.POINTER(SsdConfig), ctypes.POINTER(PrefillArgs),
                                       ctypes.POINTER(c_int), c_int, vp]
    lib.ssd_prefill_noalloc.restype = c_int
    lib.ssd_prefill_noalloc.argtypes = [ctypes.POINTER(SsdConfig), ctypes.POINTER(PrefillArgs), vp]
    lib.ssd_prefill_span_state.restype = c_int
    lib.ssd_prefill_span_state.argtypes = [ctypes.POINTER(SsdConfig), ctypes.POINTER(PrefillArgs), vp, vp, vp]
    lib.ssd_span_prefix.restype = c_int
    lib.ssd_span_prefix.argtypes = [vp, vp, c_int, c_int, c_int, c_int, c_int, vp, vp, vp, vp]
    lib.ssd_test_stall_scan.restype = None
    lib.ssd_test_stall_scan.argtypes = [c_int, ctypes.c_ulonglong]
    lib.ssd_debug_bounds_build.restype = c_int
    lib.ssd_debug_bounds_build.argtypes = []
    lib.ssd_test_bounds_scale.restype = None
    lib.ssd_test_bounds_scale.argtypes = [c_int]
    lib.ssd_trace_enable.restype = c_int
    lib.ssd_trace_enable.argtypes = [c_int]
    lib.ssd_trace_read.restype = c_int
    lib.ssd_trace_read.argtypes = [ctypes.POINTER(TraceRecord), c_int]
    _lib = lib
    return lib


# ---------------------------------------------------------------------------------------------
def make_config(cfg: dict, seqlen: int | None = None, kernel: int | None = None) -> SsdConfig:
    """C config from a workload dict (datagen.config style)."""
    dtype = cfg.get("dtype", "bf16")
    return SsdConfig(
        batch=cfg["batch"], seqlen=cfg["seqlen"] if seqlen is None else seqlen,
        nheads=cfg["nheads"], headdim=cfg.get("headdim", 64), dstate=cfg.get("dstate", 128),
        ngroups=cfg["ngroups"], chunk=cfg.get("chunk", 128), conv_width=cfg.get("conv_width", 4),
        norm_groups=cfg.get("norm_groups", 0), norm_eps=cfg.get("norm_eps", 1e-5),
        dt_min=cfg.get("dt_min", 0.0), dt_max=cfg.get("dt_max", math.inf),
        dt_softplus=int(cfg.get("dt_softplus", True)),
        io_dtype=SSD_BF16 if dtype == "bf16" else SSD_F32,
        n_segments=cfg.get("n_segments", 0),
        kernel=cfg.get("kernel", KERNEL_AUTO) if kernel is None else kernel,
        norm_before_gate=int(cfg.get("norm_before_gate", False)))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _row_stride(t, L: int | None = None) -> int:
    """Elements between consecutive rows (tokens) of a channels-contiguous tensor."""
    assert t.stride(-1) == 1, "channels must be contiguous"
    if t.dim() >= 2:
        rs = t.stride(-2)
        if t.dim() == 3 and t.shape[0] > 1 and t.shape[1] > 1:
            assert t.stride(0) == t.shape[1] * rs, "batch rows must be seqlen * row_stride apart"
        return rs
    return t.shape[-1]


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(status: int, where: str):
    if status != 0:
        raise SsdError(status, where)


def io_dtype(cfg: dict):
    import torch
    return torch.bfloat16 if cfg.get("dtype", "bf16") == "bf16" else torch.float32


def to_device(a, device="cuda", bf16=None):
    """numpy (uint16 = bf16 bits, float32) -> torch tensor on the device."""
    import torch
    if isinstance(a, torch.Tensor):
        return a.to(device)
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(a).to(device)


def to_numpy(t) -> np.ndarray:
    """torch tensor -> numpy (bf16 becomes uint16 bit patterns)."""
    import torch
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def workspace_size(cfg: dict, seqlen: int | None = None, kernel: int | None = None) -> int:
    c = make_config(cfg, seqlen, kernel)
    return load().ssd_workspace_size(ctypes.byref(c))


def varlen_workspace_size(cfg: dict, cu_seqlens, kernel: int | None = None) -> int:
    """ssd_varlen_workspace_size for the packed batch with offsets cu_seqlens."""
    cu = [int(v) for v in cu_seqlens]
    c = make_config(dict(cfg, batch=1), seqlen=cu[-1], kernel=kernel)
    return load().ssd_varlen_workspace_size(ctypes.byref(c), (c_int * len(cu))(*cu), len(cu) - 1)


def alloc_workspace(nbytes: int, device="cuda"):
    import torch
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def prefill(cfg: dict, xBC, dt, A, D, dt_bias, conv_w=None, conv_b=None, z=None, norm_w=None,
            h0=None, conv_state_in=None, *, y=None, h_final=None, conv_state_out=None,
            workspace=None, stream=None, want_state: bool = True, kernel: int | None = None):
    """ssd_prefill over the tensors given; returns (y, h_final, conv_state_out)."""
    import torch
    lib = load()
    Bn, L = xBC.shape[0], xBC.shape[1]
    c = make_config(cfg, seqlen=L, kernel=kernel)
    H, P, N, G, W = c.nheads, c.headdim, c.dstate, c.ngroups, c.conv_width
    d_inner, conv_dim = H * P, H * P + 2 * G * N
    dev = xBC.device
    if y is None:
        y = torch.empty((Bn, L, d_inner), dtype=io_dtype(cfg), device=dev)
    if h_final is None and want_state:
        h_final = torch.empty((Bn, H, P, N), dtype=torch.float32, device=dev)
    if conv_state_out is None and want_state and W > 0:
        conv_state_out = torch.empty((Bn, W, conv_dim), dtype=io_dtype(cfg), device=dev)
    if workspace is None:
        workspace = alloc_workspace(lib.ssd_workspace_size(ctypes.byref(c)), dev)
    a = PrefillArgs(
        xBC=_ptr(xBC), xBC_row_stride=_row_stride(xBC), dt=_ptr(dt), dt_row_stride=_row_stride(dt),
        z=_ptr(z), z_row_stride=_row_stride(z) if z is not None else 0, A=_ptr(A), D=_ptr(D),
        dt_bias=_ptr(dt_bias), conv_w=_ptr(conv_w), conv_b=_ptr(conv_b), norm_w=_ptr(norm_w),
        h0=_ptr(h0), conv_state_in=_ptr(conv_state_in), y=_ptr(y), y_row_stride=_row_stride(y),
        h_final=_ptr(h_final), conv_state_out=_ptr(conv_state_out), workspace=_ptr(workspace),
        workspace_bytes=workspace.numel())
    _check(lib.ssd_prefill(ctypes.byref(c), ctypes.byref(a), _stream(stream)), "ssd_prefill")
    return y, h_final, conv_state_out


def prefill_noalloc(cfg: dict, xBC, dt, A, D, dt_bias, conv_w=None, conv_b=None, z=None, norm_w=None,
                    h0=None, conv_state_in=None, *, y=None, h_final=None, conv_state_out=None,
                    stream=None, kernel: int | None = None):
    """ssd_prefill_noalloc: the same computation as prefill() with the library's fixed device
    scratch instead of a caller workspace (for callers that must not allocate device memory).
    Outputs that are not passed are allocated here by torch; the C call allocates nothing."""
    import torch
    lib = load()
    Bn, L = xBC.shape[0], xBC.shape[1]
    c = make_config(cfg, seqlen=L, kernel=kernel)
    H, P, N, G, W = c.nheads, c.headdim, c.dstate, c.ngroups, c.conv_width
    d_inner, conv_dim = H * P, H * P + 2 * G * N
    dev = xBC.device
    if y is None:
        y = torch.empty((Bn, L, d_inner), dtype=io_dtype(cfg), device=dev)
    if h_final is None:
        h_final = torch.empty((Bn, H, P, N), dtype=torch.float32, device=dev)
    if conv_state_out is None and W > 0:
        conv_state_out = torch.empty((Bn, W, conv_dim), dtype=io_dtype(cfg), device=dev)
    a = PrefillArgs(
        xBC=_ptr(xBC), xBC_row_stride=_row_stride(xBC), dt=_ptr(dt), dt_row_stride=_row_stride(dt),
        z=_ptr(z), z_row_stride=_row_stride(z) if z is not None else 0, A=_ptr(A), D=_ptr(D),
        dt_bias=_ptr(dt_bias), conv_w=_ptr(conv_w), conv_b=_ptr(conv_b), norm_w=_ptr(norm_w),
        h0=_ptr(h0), conv_state_in=_ptr(conv_state_in), y=_ptr(y), y_row_stride=_row_stride(y),
        h_final=_ptr(h_final), conv_state_out=_ptr(conv_state_out), workspace=None,
        workspace_bytes=0)
    _check(lib.ssd_prefill_noalloc(ctypes.byref(c), ctypes.byref(a), _stream(stream)),
           "ssd_prefill_noalloc")
    return y, h_final, conv_state_out


def prefill_varlen(cfg: dict, cu_seqlens, xBC, dt, A, D, dt_bias, conv_w=None, conv_b=None, z=None,
                   norm_w=None, h0=None, conv_state_in=None, *, workspace=None, stream=None,
                   want_state: bool = True, kernel: int | None = None):
    """ssd_prefill_varlen: packed sequences xBC [T, conv_dim] (T = cu_seqlens[-1]) with
    per-sequence carries [nseq, ...]; returns (y [T, d_inner], h_final [nseq, H, P, N] or None
    when want_state is False, conv_state_out [nseq, W, conv_dim] or None).  Without the final
    states the library skips the pass that computes their last chunks."""
    import torch
    lib = load()
    cu = [int(v) for v in cu_seqlens]
    nseq, T = len(cu) - 1, cu[-1]
    c = make_config(dict(cfg, batch=1), seqlen=T, kernel=kernel)
    H, P, N, G, W = c.nheads, c.headdim, c.dstate, c.ngroups, c.conv_width
    d_inner, conv_dim = H * P, H * P + 2 * G * N
    dev = xBC.device
    y = torch.empty((T, d_inner), dtype=io_dtype(cfg), device=dev)
    h_final = torch.empty((nseq, H, P, N), dtype=torch.float32, device=dev) if want_state else None
    cso = torch.empty((nseq, W, conv_dim), dtype=io_dtype(cfg), device=dev) if W > 0 else None
    cu_arr = (c_int * (nseq + 1))(*cu)
    if workspace is None:
        workspace = alloc_workspace(lib.ssd_varlen_workspace_size(ctypes.byref(c), cu_arr, nseq), dev)
    a = PrefillArgs(
        xBC=_ptr(xBC), xBC_row_stride=xBC.stride(-2), dt=_ptr(dt), dt_row_stride=dt.stride(-2),
        z=_ptr(z), z_row_stride=z.stride(-2) if z is not None else 0, A=_ptr(A), D=_ptr(D),
        dt_bias=_ptr(dt_bias), conv_w=_ptr(conv_w), conv_b=_ptr(conv_b), norm_w=_ptr(norm_w),
        h0=_ptr(h0), conv_state_in=_ptr(conv_state_in), y=_ptr(y), y_row_stride=d_inner,
        h_final=_ptr(h_final), conv_state_out=_ptr(cso), workspace=_ptr(workspace),
        workspace_bytes=workspace.numel())
    _check(lib.ssd_prefill_varlen(ctypes.byref(c), ctypes.byref(a), cu_arr, nseq, _stream(stream)),
           "ssd_prefill_varlen")
    return y, h_final, cso


def prefill_span_state(cfg: dict, xBC, dt, A, dt_bias, conv_w=None, conv_b=None, conv_state_in=None,
                       *, span_state=None, span_decay=None, workspace=None, stream=None,
                       kernel: int | None = None):
    """ssd_prefill_span_state: the state this span's tokens produce from a zero state and their
    total decay; returns (span_state [B, H, P, N], span_decay [B, H])."""
    import torch
    lib = load()
    Bn, L = xBC.shape[0], xBC.shape[1]
    c = make_config(cfg, seqlen=L, kernel=kernel)
    dev = xBC.device
    if span_state is None:
        span_state = torch.empty((Bn, c.nheads, c.headdim, c.dstate), dtype=torch.float32, device=dev)
    if span_decay is None:
        span_decay = torch.empty((Bn, c.nheads), dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = alloc_workspace(lib.ssd_workspace_size(ctypes.byref(c)), dev)
    a = PrefillArgs(
        xBC=_ptr(xBC), xBC_row_stride=_row_stride(xBC), dt=_ptr(dt), dt_row_stride=_row_stride(dt),
        A=_ptr(A), dt_bias=_ptr(dt_bias), conv_w=_ptr(conv_w), conv_b=_ptr(conv_b),
        conv_state_in=_ptr(conv_state_in), workspace=_ptr(workspace), workspace_bytes=workspace.numel())
    _check(lib.ssd_prefill_span_state(ctypes.byref(c), ctypes.byref(a), _ptr(span_state), _ptr(span_decay),
                                      _stream(stream)), "ssd_prefill_span_state")
    return span_state, span_decay


def span_prefix(span_states, span_decays, h0=None, *, h_in=None, h_final=None, want_h_in=True,
                want_h_final=True, stream=None):
    """ssd_span_prefix over gathered span states [S, B, H, P, N] and decays [S, B, H]; returns
    (h_in [S, B, H, P, N] or None, h_final [B, H, P, N] or None)."""
    import torch
    lib = load()
    S, Bn, H, P, N = span_states.shape
    if want_h_in and h_in is None:
        h_in = torch.empty_like(span_states)
    if want_h_final and h_final is None:
        h_final = torch.empty((Bn, H, P, N), dtype=torch.float32, device=span_states.device)
    _check(lib.ssd_span_prefix(_ptr(span_states), _ptr(span_decays), S, Bn, H, P, N, _ptr(h0),
                               _ptr(h_in) if want_h_in else None, _ptr(h_final) if want_h_final else None,
                               _stream(stream)), "ssd_span_prefix")
    return (h_in if want_h_in else None), (h_final if want_h_final else None)


def decode_step(cfg: dict, xBC_t, dt_t, A, D, dt_bias, conv_w, conv_b, state, conv_state_in,
                conv_state_out, z_t=None, norm_w=None, *, y=None, stream=None):
    """ssd_decode_step: state updated in place, conv_state_out written; returns y [B, d_inner]."""
    import torch
    lib = load()
    c = make_config(cfg, seqlen=1)
    d_inner = c.nheads * c.headdim
    if y is None:
        y = torch.empty((xBC_t.shape[0], d_inner), dtype=io_dtype(cfg), device=xBC_t.device)
    a = DecodeArgs(xBC=_ptr(xBC_t), xBC_row_stride=_row_stride(xBC_t), dt=_ptr(dt_t),
                   dt_row_stride=_row_stride(dt_t), z=_ptr(z_t),
                   z_row_stride=_row_stride(z_t) if z_t is not None else 0, A=_ptr(A), D=_ptr(D),
                   dt_bias=_ptr(dt_bias), conv_w=_ptr(conv_w), conv_b=_ptr(conv_b),
                   norm_w=_ptr(norm_w), state=_ptr(state), conv_state_in=_ptr(conv_state_in),
                   conv_state_out=_ptr(conv_state_out), y=_ptr(y), y_row_stride=_row_stride(y))
    _check(lib.ssd_decode_step(ctypes.byref(c), ctypes.byref(a), _stream(stream)), "ssd_decode_step")
    return y


def make_mixer_config(cfg: dict, seqlen: int | None = None, kernel: int | None = None) -> MixerConfig:
    return MixerConfig(ssd=make_config(cfg, seqlen, kernel), d_model=cfg["d_model"],
                       rms_eps=cfg.get("rms_eps", 1e-5))


def mixer_workspace_size(cfg: dict, seqlen: int | None = None, kernel: int | None = None) -> int:
    m = make_mixer_config(cfg, seqlen, kernel)
    return load().ssd_mixer_workspace_size(ctypes.byref(m))


def mixer_forward(cfg: dict, hidden, rms_w, W_in, W_out, A, D, dt_bias, conv_w, conv_b, norm_w,
                  h0=None, conv_state_in=None, *, out=None, h_final=None, conv_state_out=None,
                  workspace=None, stream=None, kernel: int | None = None):
    """mamba2_mixer_forward; returns out [B, L, d_model] bf16."""
    import torch
    lib = load()
    m = make_mixer_config(cfg, seqlen=hidden.shape[1], kernel=kernel)
    if out is None:
        out = torch.empty(hidden.shape, dtype=torch.bfloat16, device=hidden.device)
    if workspace is None:
        workspace = alloc_workspace(lib.ssd_mixer_workspace_size(ctypes.byref(m)), hidden.device)
    a = MixerArgs(hidden=_ptr(hidden), rms_w=_ptr(rms_w), W_in=_ptr(W_in), W_out=_ptr(W_out),
                  A=_ptr(A), D=_ptr(D), dt_bias=_ptr(dt_bias), conv_w=_ptr(conv_w),
                  conv_b=_ptr(conv_b), norm_w=_ptr(norm_w), h0=_ptr(h0),
                  conv_state_in=_ptr(conv_state_in), h_final=_ptr(h_final),
                  conv_state_out=_ptr(conv_state_out), out=_ptr(out), workspace=_ptr(workspace),
                  workspace_bytes=workspace.numel())
    _check(lib.mamba2_mixer_forward(ctypes.byref(m), ctypes.byref(a), _stream(stream)),
           "mamba2_mixer_forward")
    return out


def get_device_error(stream=None) -> int:
    """Waits for the stream, returns and clears the library's device error status."""
    return load().ssd_get_device_error(_stream(stream))


def test_stall_scan(chunk: int, wait_limit_ms: float = 20.0) -> None:
    """Test hook: tensor-core prefills withhold chunk `chunk`'s stage so that their bounded
    waits give up after wait_limit_ms (SSD_ERR_TIMEOUT); chunk < 0 turns it off."""
    load().ssd_test_stall_scan(int(chunk), int(wait_limit_ms * 1e6))


def trace_enable(on: bool) -> bool:
    """Bracket every library kernel launch with CUDA events (for measurement); returns the
    previous setting."""
    return bool(load().ssd_trace_enable(int(on)))


def trace_read(max_records: int = 1 << 16) -> list[tuple[str, float]]:
    """(kernel name, milliseconds) of every traced launch since the last read, oldest first."""
    buf = (TraceRecord * max_records)()
    n = load().ssd_trace_read(buf, max_records)
    if n < 0:
        raise SsdError(4, "ssd_trace_read")
    return [(buf[i].name.decode(), float(buf[i].ms)) for i in range(n)]
