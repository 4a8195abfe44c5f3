"""fp64 CPU oracle for the Mamba-2 selective-scan hot path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg import this package.  The CUDA library never
calls it, and it never imports the CUDA library: the two share nothing except
the seeded input generators, which hold none of the method's arithmetic.

The arithmetic lives in ``ssd_oracle.c`` (plain sequential loops in fp64).  This
module compiles it with gcc, marshals numpy arrays to it, and composes the
steps of the mixer exactly in the order the method defines them:

  conv1d(window 4) + SiLU on the x|B|C channels, softplus dt,
  h_t = exp(dt_t A_h) h_{t-1} + dt_t x_t B_t^T,  y_t = h_t C_t + D_h x_t,
  then the z-gated RMSNorm y*silu(z) normalised per group of channels.

The hyper-parameters (8 groups, state 128, head dim 64, expansion 2, conv
window 4, RMSNorm, no linear bias) are those of the Mamba-2 layers in the
"NVIDIA Nemotron Nano 2" pages (hyper.ai summary, section "Method";
neurohive.io article, section "Model architecture"); the fp32 SSM cache
requirement is from the neurohive.io article, section "Deployment and usage".

Also here: ``quadratic_form``, the brute-force materialised form
y = (L o C B^T) X + (decayed h0 read-out) + D x of the same scan, written
independently of the recurrence for the CPU pins.

Arrays: float64 / float32 arrays are read as such; uint16 arrays are bf16 bit
patterns (read exactly).  Outputs are float64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import tempfile

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssd_oracle.c")
DEFAULT_LIB = os.path.join(_HERE, "liboracle.so")

_F64, _F32, _BF16 = 0, 1, 2


def compile_oracle(out_path: str = DEFAULT_LIB, mutant: int = 0) -> str:
    """Compile ssd_oracle.c into a shared library (gcc, -O2, no fast-math)."""
    cmd = ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11", f"-DORACLE_MUTANT={mutant}",
           "-o", out_path, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    return out_path


class _Shape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("seqlen", ctypes.c_int), ("nheads", ctypes.c_int),
                ("headdim", ctypes.c_int), ("dstate", ctypes.c_int), ("ngroups", ctypes.c_int),
                ("conv_width", ctypes.c_int), ("dt_softplus", ctypes.c_int),
                ("dt_min", ctypes.c_double), ("dt_max", ctypes.c_double)]


def _code(a: np.ndarray) -> int:
    if a.dtype == np.float64:
        return _F64
    if a.dtype == np.float32:
        return _F32
    if a.dtype == np.uint16:
        return _BF16
    raise TypeError(f"unsupported oracle input dtype {a.dtype}")


def _p(a):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"] or a.ndim == 0
    return a.ctypes.data_as(ctypes.c_void_p)


def _as_param(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    return a if a.dtype in (np.float64, np.float32, np.uint16) else a.astype(np.float64)


def bf16_to_f64(u16: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float64."""
    return (u16.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def to_f64(a: np.ndarray) -> np.ndarray:
    return bf16_to_f64(a) if a.dtype == np.uint16 else np.asarray(a, dtype=np.float64)


class Oracle:
    """Bindings to one build of ssd_oracle.c (the default build, or a planted mutant)."""

    def __init__(self, lib_path: str = DEFAULT_LIB):
        if not os.path.exists(lib_path) or (lib_path == DEFAULT_LIB and
                                            os.path.getmtime(lib_path) < os.path.getmtime(_SRC)):
            compile_oracle(lib_path)
        self.lib = ctypes.CDLL(lib_path)
        L = self.lib
        L.oracle_round_bf16.restype = ctypes.c_double
        L.oracle_round_bf16.argtypes = [ctypes.c_double]
        L.oracle_silu.restype = ctypes.c_double
        L.oracle_silu.argtypes = [ctypes.c_double]
        L.oracle_softplus.restype = ctypes.c_double
        L.oracle_softplus.argtypes = [ctypes.c_double]
        L.oracle_dt.restype = ctypes.c_double
        L.oracle_dt.argtypes = [ctypes.c_double, ctypes.c_double, ctypes.c_int, ctypes.c_double,
                                ctypes.c_double]
        vp, ci, cll, cd = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_double
        L.oracle_conv1d_silu.restype = None
        L.oracle_conv1d_silu.argtypes = [ci, ci, ci, ci, vp, ci, cll, vp, ci, vp, ci, vp, ci, vp]
        L.oracle_ssd_prefill.restype = None
        L.oracle_ssd_prefill.argtypes = [ctypes.POINTER(_Shape), vp, ci, cll, vp, ci, cll, vp, vp,
                                         vp, ci, vp, vp, ci, vp, ci, vp, ci, ci, ci, vp, vp, ci]
        L.oracle_gated_rmsnorm.restype = None
        L.oracle_gated_rmsnorm.argtypes = [cll, ci, ci, vp, vp, ci, cll, vp, ci, cd, ci, vp]
        L.oracle_rmsnorm.restype = None
        L.oracle_rmsnorm.argtypes = [cll, ci, vp, ci, vp, ci, cd, vp]
        L.oracle_decode_step.restype = None
        L.oracle_decode_step.argtypes = [ctypes.POINTER(_Shape), vp, ci, vp, ci, vp, vp, vp, ci,
                                         vp, vp, ci, vp, ci, vp, vp, ci, ci, vp, ci]

    # ---- scalar helpers -------------------------------------------------------------------
    def round_bf16(self, x: float) -> float:
        return self.lib.oracle_round_bf16(float(x))

    def round_bf16_array(self, a: np.ndarray) -> np.ndarray:
        """Elementwise nearest-bf16 rounding (ties to even) of a float64 array."""
        f = np.vectorize(self.lib.oracle_round_bf16, otypes=[np.float64])
        return f(np.asarray(a, np.float64))

    def silu(self, x: float) -> float:
        return self.lib.oracle_silu(float(x))

    def softplus(self, x: float) -> float:
        return self.lib.oracle_softplus(float(x))

    def dt(self, dt_raw: float, bias: float, softplus: bool = True, dt_min: float = 0.0,
           dt_max: float = float("inf")) -> float:
        return self.lib.oracle_dt(float(dt_raw), float(bias), int(softplus), float(dt_min),
                                  float(dt_max))

    # ---- front end ------------------------------------------------------------------------
    def conv1d_silu(self, xin: np.ndarray, w: np.ndarray, bias=None, state_in=None) -> np.ndarray:
        """u[b,t,c] = silu(bias_c + sum_k w[c,k] xin[b, t-(W-1)+k, c]) with history from
        state_in [B, W, C] (zeros when None).  xin [B, L, C]; w [C, W]."""
        xin = np.ascontiguousarray(xin)
        Bn, L, C = xin.shape
        W = w.shape[1]
        w = _as_param(w)
        bias = None if bias is None else _as_param(bias)
        state_in = None if state_in is None else np.ascontiguousarray(state_in)
        u = np.empty((Bn, L, C), np.float64)
        self.lib.oracle_conv1d_silu(Bn, L, C, W, _p(xin), _code(xin), C, _p(state_in),
                                    _code(state_in) if state_in is not None else 0, _p(w),
                                    _code(w), _p(bias), _code(bias) if bias is not None else 0,
                                    _p(u))
        return u

    # ---- prefill ----------------------------------------------------------------------------
    def ssd_prefill(self, cfg: dict, xBC: np.ndarray, dt: np.ndarray, A, D, dt_bias, conv_w=None,
                    conv_b=None, h0=None, conv_state_in=None, z=None, norm_w=None, heads=None,
                    threads: int | None = None) -> dict:
        """Plain recurrence over heads [lo, hi) of every batch row.

        cfg keys: batch, seqlen, nheads, headdim, dstate, ngroups, conv_width (0 = no conv),
        dt_softplus (bool), dt_min, dt_max, norm_groups (0 = no gate/norm), norm_eps.
        xBC [B, L, >= conv_dim] (x|B|C in the first conv_dim columns), dt [B, L, >= H].
        Returns y (pre-gate, [B, L, nh, P]), h_final [B, nh, P, N], and when norm_groups > 0
        ``out`` = gated RMSNorm of y ([B, L, nh*P]); heads must then cover whole norm groups.
        conv_state_out [B, W, conv_dim] (raw inputs, input dtype) is returned when lo == 0.
        """
        Bn, L, H, P, N, G = (cfg["batch"], cfg["seqlen"], cfg["nheads"], cfg["headdim"],
                             cfg["dstate"], cfg["ngroups"])
        W = cfg.get("conv_width", 4)
        lo, hi = heads if heads is not None else (0, H)
        conv_dim = H * P + 2 * G * N
        shape = _Shape(Bn, L, H, P, N, G, W, int(cfg.get("dt_softplus", True)),
                       float(cfg.get("dt_min", 0.0)), float(cfg.get("dt_max", np.inf)))
        xBC, dt = np.ascontiguousarray(xBC), np.ascontiguousarray(dt)
        xs, ds = xBC.shape[-1], dt.shape[-1]
        A, D, dt_bias = to_f64(A).copy(), to_f64(D).copy(), to_f64(dt_bias).copy()
        if W > 0:
            conv_w = np.ascontiguousarray(to_f64(conv_w))
            if conv_b is not None:
                conv_b = np.ascontiguousarray(to_f64(conv_b))
        nh = hi - lo
        y = np.empty((Bn, L, nh, P), np.float64)
        hf = np.empty((Bn, nh, P, N), np.float64)
        h0c = None if h0 is None else np.ascontiguousarray(h0)
        csi = None if conv_state_in is None else np.ascontiguousarray(conv_state_in)
        self.lib.oracle_ssd_prefill(
            ctypes.byref(shape), _p(xBC), _code(xBC), xs, _p(dt), _code(dt), ds, _p(A), _p(D),
            _p(dt_bias), _F64, _p(conv_w) if W > 0 else None,
            _p(conv_b) if (W > 0 and conv_b is not None) else None, _F64, _p(h0c), _code(h0c) if h0c is not None else 0,
            _p(csi), _code(csi) if csi is not None else 0, lo, hi, _p(y), _p(hf),
            int(threads if threads else (os.cpu_count() or 1)))
        res = {"y": y, "h_final": hf}
        ng = cfg.get("norm_groups", 0)
        if ng:
            gs = H * P // ng
            assert (lo * P) % gs == 0 and (hi * P) % gs == 0, "heads must cover whole norm groups"
            zz = None if z is None else z[..., lo * P:hi * P]
            res["out"] = self.gated_rmsnorm(
                y.reshape(Bn * L, nh * P), None if z is None else
                np.ascontiguousarray(zz).reshape(Bn * L, nh * P),
                None if norm_w is None else np.ascontiguousarray(norm_w)[lo * P:hi * P],
                ngroups=nh * P // gs, eps=cfg.get("norm_eps", 1e-5),
                norm_before_gate=cfg.get("norm_before_gate", False)).reshape(Bn, L, nh * P)
        if lo == 0 and W > 0:
            raw = xBC.reshape(Bn, L, -1)[:, :, :conv_dim]
            res["conv_state_out"] = self.conv_state_after(raw, conv_state_in, W)
        return res

    @staticmethod
    def conv_state_after(raw: np.ndarray, conv_state_in, W: int) -> np.ndarray:
        """The last W raw inputs of (cache ++ sequence), oldest first, in the input dtype."""
        Bn, L, C = raw.shape
        hist = conv_state_in if conv_state_in is not None else np.zeros((Bn, W, C), raw.dtype)
        return np.ascontiguousarray(np.concatenate([hist.astype(raw.dtype), raw], axis=1)[:, -W:])

    # ---- norms ------------------------------------------------------------------------------
    def gated_rmsnorm(self, y: np.ndarray, z, w, ngroups: int, eps: float = 1e-5,
                      norm_before_gate: bool = False) -> np.ndarray:
        y = np.ascontiguousarray(y, dtype=np.float64)
        T, Dn = y.shape
        z = None if z is None else np.ascontiguousarray(z)
        w = None if w is None else _as_param(w)
        out = np.empty_like(y)
        self.lib.oracle_gated_rmsnorm(T, Dn, ngroups, _p(y), _p(z), _code(z) if z is not None else 0,
                                      Dn, _p(w), _code(w) if w is not None else 0, float(eps),
                                      int(bool(norm_before_gate)), _p(out))
        return out

    def rmsnorm(self, x: np.ndarray, w, eps: float = 1e-5) -> np.ndarray:
        x = np.ascontiguousarray(x)
        T, Dn = x.shape
        w = None if w is None else _as_param(w)
        out = np.empty((T, Dn), np.float64)
        self.lib.oracle_rmsnorm(T, Dn, _p(x), _code(x), _p(w), _code(w) if w is not None else 0,
                                float(eps), _p(out))
        return out

    # ---- decode -----------------------------------------------------------------------------
    def decode_step(self, cfg: dict, xBC_t, dt_t, A, D, dt_bias, conv_w, conv_b, conv_state_in,
                    state: np.ndarray, z_t=None, norm_w=None, heads=None,
                    threads: int | None = None) -> dict:
        """One token per batch row.  ``state`` [B, nh, P, N] float64 is updated in place.
        Returns y (pre-gate [B, nh, P]), out (gated norm, if norm_groups), conv_state_out."""
        Bn, H, P, N, G = cfg["batch"], cfg["nheads"], cfg["headdim"], cfg["dstate"], cfg["ngroups"]
        W = cfg.get("conv_width", 4)
        lo, hi = heads if heads is not None else (0, H)
        conv_dim = H * P + 2 * G * N
        shape = _Shape(Bn, 1, H, P, N, G, W, int(cfg.get("dt_softplus", True)),
                       float(cfg.get("dt_min", 0.0)), float(cfg.get("dt_max", np.inf)))
        assert state.dtype == np.float64 and state.flags["C_CONTIGUOUS"]
        A, D, dt_bias = to_f64(A).copy(), to_f64(D).copy(), to_f64(dt_bias).copy()
        conv_w = np.ascontiguousarray(to_f64(conv_w))
        if conv_b is not None:
            conv_b = np.ascontiguousarray(to_f64(conv_b))
        xBC_t, dt_t = np.ascontiguousarray(xBC_t), np.ascontiguousarray(dt_t)
        csi = np.ascontiguousarray(conv_state_in)
        cso = np.empty((Bn, max(W, 1), conv_dim), np.float64)
        nh = hi - lo
        y = np.empty((Bn, nh, P), np.float64)
        self.lib.oracle_decode_step(ctypes.byref(shape), _p(xBC_t), _code(xBC_t), _p(dt_t),
                                    _code(dt_t), _p(A), _p(D), _p(dt_bias), _F64, _p(conv_w),
                                    _p(conv_b), _F64, _p(csi), _code(csi), _p(cso),
                                    _p(state), lo, hi, _p(y),
                                    int(threads if threads else (os.cpu_count() or 1)))
        res = {"y": y, "conv_state_out": cso}
        ng = cfg.get("norm_groups", 0)
        if ng:
            zz = np.ascontiguousarray(z_t[:, lo * P:hi * P])
            gs = H * P // ng
            res["out"] = self.gated_rmsnorm(
                y.reshape(Bn, nh * P), zz,
                None if norm_w is None else np.ascontiguousarray(norm_w)[lo * P:hi * P],
                ngroups=nh * P // gs, eps=cfg.get("norm_eps", 1e-5),
                norm_before_gate=cfg.get("norm_before_gate", False))
        return res

    # ---- full mixer layer ---------------------------------------------------------------------
    def mixer_forward(self, cfg: dict, hidden, rms_w, W_in, W_out, A, D, dt_bias, conv_w, conv_b,
                      norm_w, rows=None, tokens=None, threads=None,
                      bf16_activations: bool = True) -> np.ndarray:
        """RMSNorm -> in_proj -> (z | xBC | dt) -> conv/SiLU + scan + gated RMSNorm -> out_proj.

        hidden [B, L, d_model]; W_in [2*d_inner + 2GN + H, d_model]; W_out [d_model, d_inner].
        ``rows`` selects batch rows and ``tokens`` a causal prefix length (both exact, because
        rows are independent and the layer is causal).  Returns out [len(rows), tokens, d_model].

        The layer runs in bf16 ("bfloat16 precision", Nemotron Nano 2 abstract): with
        ``bf16_activations`` the three activation tensors the layer materialises between its
        steps (RMSNorm output, in_proj output, gated-norm output) are rounded to bf16; all
        arithmetic is fp64 otherwise.
        """
        Bn, L, H, P, N, G = (cfg["batch"], cfg["seqlen"], cfg["nheads"], cfg["headdim"],
                             cfg["dstate"], cfg["ngroups"])
        rows = list(range(Bn)) if rows is None else list(rows)
        T = L if tokens is None else tokens
        d_model = cfg["d_model"]
        d_inner = H * P
        hid = np.ascontiguousarray(hidden[rows][:, :T])
        rnd = self._round_bf16_fast if bf16_activations else (lambda v: v)
        hn = rnd(self.rmsnorm(hid.reshape(-1, d_model), rms_w, eps=cfg.get("rms_eps", 1e-5)))
        zxbcdt = rnd(hn @ to_f64(W_in).T)  # library matmul in fp64
        zxbcdt = zxbcdt.reshape(len(rows), T, -1)
        conv_dim = d_inner + 2 * G * N
        z = np.ascontiguousarray(zxbcdt[..., :d_inner])
        xBC = np.ascontiguousarray(zxbcdt[..., d_inner:d_inner + conv_dim])
        dt = np.ascontiguousarray(zxbcdt[..., d_inner + conv_dim:])
        c2 = dict(cfg, batch=len(rows), seqlen=T)
        r = self.ssd_prefill(c2, xBC, dt, A, D, dt_bias, conv_w=conv_w, conv_b=conv_b, z=z,
                             norm_w=norm_w, threads=threads)
        g = rnd(r["out"].reshape(-1, d_inner))
        return (g @ to_f64(W_out).T).reshape(len(rows), T, d_model)

    @staticmethod
    def _round_bf16_fast(a: np.ndarray) -> np.ndarray:
        """Vectorised nearest-bf16 rounding, ties to even, from float64 (same definition as
        oracle_round_bf16: keep 8 significant bits of the binary mantissa)."""
        a = np.asarray(a, np.float64)
        m, e = np.frexp(a)
        return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)


def quadratic_form(x, Bm, Cm, dt, A, D, h0=None) -> np.ndarray:
    """Brute-force materialised SSD (no conv, no gate), fp64, small sizes only.

    For each batch row and head (group g = h // (H/G)):
      M[t, s] = (C_t . B_s) * exp(A_h * sum_{r=s+1..t} dt_r) * dt_s   for s <= t, else 0
      y_t = sum_s M[t, s] x_s + exp(A_h * sum_{r<=t} dt_r) * (h0 C_t) + D_h x_t
    x [Bt, L, H, P]; Bm, Cm [Bt, L, G, N]; dt [Bt, L, H] (already the effective step);
    h0 [Bt, H, P, N] or None.  Returns y [Bt, L, H, P].
    """
    x, Bm, Cm, dt = (np.asarray(a, np.float64) for a in (x, Bm, Cm, dt))
    A, D = np.asarray(A, np.float64), np.asarray(D, np.float64)
    Bt, L, H, P = x.shape
    G = Bm.shape[2]
    hpg = H // G
    y = np.zeros_like(x)
    for b in range(Bt):
        for h in range(H):
            g = h // hpg
            M = np.zeros((L, L))
            for t in range(L):
                for s in range(t + 1):
                    seg = dt[b, s + 1:t + 1, h].sum()
                    M[t, s] = (Cm[b, t, g] @ Bm[b, s, g]) * np.exp(A[h] * seg) * dt[b, s, h]
            y[b, :, h] = M @ x[b, :, h] + D[h] * x[b, :, h]
            if h0 is not None:
                for t in range(L):
                    decay = np.exp(A[h] * dt[b, :t + 1, h].sum())
                    y[b, t, h] += decay * (np.asarray(h0, np.float64)[b, h] @ Cm[b, t, g])
    return y


_default: Oracle | None = None


def get() -> Oracle:
    """The default oracle build (compiled on first use)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def build() -> str:
    """Compile the default oracle library (used by the package build step)."""
    return compile_oracle(DEFAULT_LIB)


def mutant(k: int, workdir: str | None = None) -> Oracle:
    """A build of the oracle with planted mistake number k (for the pin-strength tests)."""
    d = workdir or tempfile.mkdtemp(prefix="oracle_mutant_")
    return Oracle(compile_oracle(os.path.join(d, f"liboracle_m{k}.so"), mutant=k))
