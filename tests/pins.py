"""Pins of the fp64 oracle against things other than itself.

Each ``pin_*`` takes an oracle build and returns (ok, detail).  The pytest file
asserts every pin on the real oracle, and re-runs them on builds with planted
mistakes to show that each mistake fails at least one pin.

References used here are independent of the oracle's recurrence:
  - the brute-force quadratic form y = (L o C B^T) X + ... (oracle.quadratic_form,
    numpy, written from the definition of the matrix form);
  - numpy.cumsum (A = 0 reduces the scan to prefix sums);
  - the geometric-series closed form (constant dt, A, x = B = C = 1);
  - a chunked fp64 evaluation of the same scan (written below);
  - identities of SiLU / softplus, conv impulse responses, norm invariants.
"""
from __future__ import annotations

import math

import numpy as np

import oracle as _oracle
from oracle import quadratic_form


def _rng(seed):
    return np.random.default_rng(seed)


def _raw_cfg(B, L, H, G, P, N, W=0, softplus=False, dt_min=0.0, dt_max=math.inf, norm_groups=0):
    return dict(batch=B, seqlen=L, nheads=H, headdim=P, dstate=N, ngroups=G, conv_width=W,
                dt_softplus=softplus, dt_min=dt_min, dt_max=dt_max, norm_groups=norm_groups,
                norm_eps=1e-5)


def _split(xBC, H, P, G, N):
    Bt, L, _ = xBC.shape
    d = H * P
    x = xBC[..., :d].reshape(Bt, L, H, P)
    Bm = xBC[..., d:d + G * N].reshape(Bt, L, G, N)
    Cm = xBC[..., d + G * N:d + 2 * G * N].reshape(Bt, L, G, N)
    return x, Bm, Cm


def _rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    den = max(np.sqrt(np.mean(b * b)), 1e-300)
    return float(np.max(np.abs(a - b)) / den)


def chunked_scan(x, Bm, Cm, dt, A, D, h0, Q):
    """fp64 chunked evaluation: per chunk, intra-chunk (L o C B^T) X, decayed read-out of the
    incoming state, then the chunk's state update.  Same result as the recurrence up to
    rounding for any chunk length Q."""
    Bt, L, H, P = x.shape
    G, N = Bm.shape[2], Bm.shape[3]
    hpg = H // G
    y = np.zeros_like(x)
    hf = np.zeros((Bt, H, P, N))
    for b in range(Bt):
        for h in range(H):
            g = h // hpg
            st = np.zeros((P, N)) if h0 is None else np.array(h0[b, h], np.float64)
            for c0 in range(0, L, Q):
                sl = slice(c0, min(L, c0 + Q))
                d = dt[b, sl, h]
                cs = np.cumsum(d * A[h])
                q = len(d)
                Lm = np.zeros((q, q))
                for t in range(q):
                    for s in range(t + 1):
                        Lm[t, s] = math.exp(cs[t] - cs[s]) * d[s]
                S = Cm[b, sl, g] @ Bm[b, sl, g].T
                y[b, sl, h] = ((S * Lm) @ x[b, sl, h] + np.exp(cs)[:, None] * (Cm[b, sl, g] @ st.T)
                               + D[h] * x[b, sl, h])
                w = np.exp(cs[-1] - cs) * d
                st = math.exp(cs[-1]) * st + (x[b, sl, h] * w[:, None]).T @ Bm[b, sl, g]
            hf[b, h] = st
    return y, hf


# ---------------------------------------------------------------------------------------------
def pin_activation_identities(o):
    xs = [-7.5, -1.0, -0.25, 0.0, 0.3, 2.0, 11.0]
    bad = []
    for v in xs:
        if abs((o.silu(v) - o.silu(-v)) - v) > 1e-14 * max(1, abs(v)):
            bad.append(f"silu({v})")  # x*s(x) - (-x)*s(-x) = x
        if abs((o.softplus(v) - o.softplus(-v)) - v) > 1e-14 * max(1, abs(v)):
            bad.append(f"softplus({v})")  # log(1+e^x) - log(1+e^-x) = x
    if abs(o.softplus(0.0) - math.log(2.0)) > 1e-15:
        bad.append("softplus(0) != ln 2")
    if abs(o.silu(1.0) - 1.0 / (1.0 + math.exp(-1.0))) > 1e-15:
        bad.append("silu(1) != sigmoid(1)")
    if abs(o.softplus(50.0) - 50.0) > 1e-15 or o.softplus(800.0) != 800.0:
        bad.append("softplus large-x")
    if o.dt(-30.0, 0.0, True, 1e-3, 1e-1) != 1e-3 or o.dt(30.0, 0.0, True, 1e-3, 1e-1) != 1e-1:
        bad.append("dt clamp")
    if o.dt(0.02, 0.01, False) != 0.02 + 0.01:
        bad.append("dt without softplus")
    return (not bad), ",".join(bad)


def pin_quadratic_form(o, seed=1):
    """P1: recurrence == brute-force (L o C B^T) X form, random h0, G=2 of 4 heads."""
    r = _rng(seed)
    B, L, H, G, P, N = 2, 29, 4, 2, 3, 5
    cfg = _raw_cfg(B, L, H, G, P, N)
    xBC = r.standard_normal((B, L, H * P + 2 * G * N))
    dt = r.uniform(0.01, 0.3, (B, L, H))
    A = -r.uniform(0.5, 3.0, H)
    D = r.uniform(0, 1, H)
    h0 = r.standard_normal((B, H, P, N))
    res = o.ssd_prefill(cfg, xBC, dt, A, D, np.zeros(H), h0=h0, threads=1)
    x, Bm, Cm = _split(xBC, H, P, G, N)
    yq = quadratic_form(x, Bm, Cm, dt, A, D, h0)
    e = _rel(res["y"], yq)
    return e < 1e-12, f"rel err {e:.2e}"


def pin_quadratic_with_conv(o, seed=2):
    """P1 through the front end: conv+SiLU outputs and softplus/clamped dt fed to the
    quadratic form reproduce the composed prefill."""
    r = _rng(seed)
    B, L, H, G, P, N, W = 1, 23, 4, 2, 2, 3, 4
    cfg = _raw_cfg(B, L, H, G, P, N, W=W, softplus=True, dt_min=1e-3, dt_max=0.2)
    C = H * P + 2 * G * N
    xBC = r.standard_normal((B, L, C))
    dtr = r.standard_normal((B, L, H))
    bias = r.uniform(-4, -1, H)
    A, D = -r.uniform(0.5, 3.0, H), r.uniform(0, 1, H)
    cw, cb = r.normal(0, 0.5, (C, W)), r.normal(0, 0.1, C)
    csi = r.standard_normal((B, W, C))
    res = o.ssd_prefill(cfg, xBC, dtr, A, D, bias, conv_w=cw, conv_b=cb, conv_state_in=csi,
                        threads=1)
    u = o.conv1d_silu(xBC, cw, cb, csi)
    dte = np.vectorize(lambda v, h: o.dt(v, bias[h], True, 1e-3, 0.2))(
        dtr, np.arange(H)[None, None, :])
    x, Bm, Cm = _split(u, H, P, G, N)
    e = _rel(res["y"], quadratic_form(x, Bm, Cm, dte, A, D))
    return e < 1e-12, f"rel err {e:.2e}"


def pin_prefix_sum(o, seed=3):
    """P2: A = 0, P = N = 1, B = C = 1, D = 0 => y_t = sum_{s<=t} dt_s x_s (numpy cumsum);
    general shapes: h_final = sum_s dt_s x_s B_s^T."""
    r = _rng(seed)
    L = 41
    x = r.standard_normal(L)
    dt = r.uniform(0.01, 0.5, L)
    xBC = np.stack([x, np.ones(L), np.ones(L)], -1)[None]
    res = o.ssd_prefill(_raw_cfg(1, L, 1, 1, 1, 1), xBC, dt[None, :, None], np.zeros(1),
                        np.zeros(1), np.zeros(1), threads=1)
    e1 = _rel(res["y"][0, :, 0, 0], np.cumsum(dt * x))
    B, H, G, P, N = 2, 4, 2, 3, 4
    xBC = r.standard_normal((B, L, H * P + 2 * G * N))
    dt = r.uniform(0.01, 0.5, (B, L, H))
    res = o.ssd_prefill(_raw_cfg(B, L, H, G, P, N), xBC, dt, np.zeros(H), np.zeros(H),
                        np.zeros(H), threads=1)
    xx, Bm, _ = _split(xBC, H, P, G, N)
    Bh = np.repeat(Bm, H // G, axis=2)
    ref = np.einsum("blh,blhp,blhn->bhpn", dt, xx, Bh)
    e2 = _rel(res["h_final"], ref)
    return max(e1, e2) < 1e-12, f"rel err {e1:.2e} {e2:.2e}"


def pin_zero_dt(o, seed=4):
    """P3: dt = 0 => h stays h0, y = D x + h0 C_t; with h0 = 0, y = D x exactly."""
    r = _rng(seed)
    B, L, H, G, P, N = 2, 9, 4, 2, 3, 5
    xBC = r.standard_normal((B, L, H * P + 2 * G * N))
    A, D = -r.uniform(0.5, 3, H), r.uniform(0, 1, H)
    h0 = r.standard_normal((B, H, P, N))
    zero = np.zeros((B, L, H))
    res = o.ssd_prefill(_raw_cfg(B, L, H, G, P, N), xBC, zero, A, D, np.zeros(H), h0=h0,
                        threads=1)
    x, _, Cm = _split(xBC, H, P, G, N)
    Ch = np.repeat(Cm, H // G, axis=2)
    ref = D[None, None, :, None] * x + np.einsum("bhpn,blhn->blhp", h0, Ch)
    e = _rel(res["y"], ref)
    ok = e < 1e-13 and np.array_equal(res["h_final"], h0)
    res0 = o.ssd_prefill(_raw_cfg(B, L, H, G, P, N), xBC, zero, A, D, np.zeros(H), threads=1)
    ok = ok and np.array_equal(res0["y"], D[None, None, :, None] * x)
    return ok, f"rel err {e:.2e}"


def pin_geometric(o):
    """P4: constant dt, A; x = B = C = 1; P = N = 1; h0 = 0 =>
    h_t = dt (1 - a^{t+1}) / (1 - a), a = e^{dt A}; y_t = h_t + D."""
    L, dt, A, D = 200, 0.07, -1.3, 0.4
    xBC = np.ones((1, L, 3))
    res = o.ssd_prefill(_raw_cfg(1, L, 1, 1, 1, 1), xBC, np.full((1, L, 1), dt), np.array([A]),
                        np.array([D]), np.zeros(1), threads=1)
    a = math.exp(dt * A)
    t = np.arange(L)
    h = dt * (1 - a ** (t + 1)) / (1 - a)
    e = _rel(res["y"][0, :, 0, 0], h + D)
    e2 = abs(res["h_final"][0, 0, 0, 0] - h[-1]) / h[-1]
    return max(e, e2) < 1e-12, f"rel err {e:.2e} {e2:.2e}"


def pin_chunk_invariance(o, seed=5):
    """P5: the chunked form at Q in {1, 16, 64, L} equals the recurrence."""
    r = _rng(seed)
    B, L, H, G, P, N = 1, 70, 4, 2, 3, 4
    xBC = r.standard_normal((B, L, H * P + 2 * G * N))
    dt = r.uniform(0.01, 0.2, (B, L, H))
    A, D = -r.uniform(1, 16, H), r.uniform(0, 1, H)
    h0 = r.standard_normal((B, H, P, N))
    res = o.ssd_prefill(_raw_cfg(B, L, H, G, P, N), xBC, dt, A, D, np.zeros(H), h0=h0, threads=1)
    x, Bm, Cm = _split(xBC, H, P, G, N)
    worst = 0.0
    for Q in (1, 16, 64, L):
        yc, hc = chunked_scan(x, Bm, Cm, dt, A, D, h0, Q)
        worst = max(worst, _rel(res["y"], yc), _rel(res["h_final"], hc))
    return worst < 1e-12, f"rel err {worst:.2e}"


def pin_split_carry(o, seed=6):
    """P6: prefill(L) == prefill(L1) -> carry (h, conv cache) -> prefill(L - L1), for L1 < W too;
    the carried conv cache is the last W raw inputs, bit-exact."""
    r = _rng(seed)
    B, L, H, G, P, N, W = 2, 19, 4, 2, 2, 3, 4
    cfg = _raw_cfg(B, L, H, G, P, N, W=W, softplus=True, dt_min=1e-3, dt_max=0.3,
                   norm_groups=2)
    C = H * P + 2 * G * N
    xBC = r.standard_normal((B, L, C)).astype(np.float32)
    dtr = r.standard_normal((B, L, H)).astype(np.float32)
    z = r.standard_normal((B, L, H * P)).astype(np.float32)
    bias, A, D = r.uniform(-4, -1, H), -r.uniform(1, 8, H), r.uniform(0, 1, H)
    cw = r.normal(0, 0.5, (C, W)).astype(np.float32)
    nw = r.uniform(0.5, 1.5, H * P)
    csi = r.standard_normal((B, W, C)).astype(np.float32)
    full = o.ssd_prefill(cfg, xBC, dtr, A, D, bias, conv_w=cw, conv_state_in=csi, z=z, norm_w=nw,
                         threads=1)
    worst, exact = 0.0, True
    for L1 in (1, 2, 3, 4, 11):
        c1 = dict(cfg, seqlen=L1)
        c2 = dict(cfg, seqlen=L - L1)
        a = o.ssd_prefill(c1, xBC[:, :L1], dtr[:, :L1], A, D, bias, conv_w=cw, conv_state_in=csi,
                          z=z[:, :L1], norm_w=nw, threads=1)
        b = o.ssd_prefill(c2, xBC[:, L1:], dtr[:, L1:], A, D, bias, conv_w=cw, h0=a["h_final"],
                          conv_state_in=a["conv_state_out"], z=z[:, L1:], norm_w=nw, threads=1)
        worst = max(worst, _rel(np.concatenate([a["out"], b["out"]], 1), full["out"]),
                    _rel(b["h_final"], full["h_final"]))
        exact = exact and np.array_equal(b["conv_state_out"], full["conv_state_out"])
    exact = exact and np.array_equal(full["conv_state_out"], xBC[:, -W:])
    return worst < 1e-12 and exact, f"rel err {worst:.2e} conv cache exact={exact}"


def pin_decode_equals_prefill(o, seed=7):
    """P7: k single-token decode steps from a carried state equal the prefill of those tokens."""
    r = _rng(seed)
    B, L0, k, H, G, P, N, W = 2, 6, 5, 4, 2, 2, 3, 4
    cfg = _raw_cfg(B, L0 + k, H, G, P, N, W=W, softplus=True, dt_min=1e-3, dt_max=0.3,
                   norm_groups=2)
    C = H * P + 2 * G * N
    xBC = r.standard_normal((B, L0 + k, C))
    dtr = r.standard_normal((B, L0 + k, H))
    z = r.standard_normal((B, L0 + k, H * P))
    bias, A, D = r.uniform(-4, -1, H), -r.uniform(1, 8, H), r.uniform(0, 1, H)
    cw, cb = r.normal(0, 0.5, (C, W)), r.normal(0, 0.1, C)
    nw = r.uniform(0.5, 1.5, H * P)
    full = o.ssd_prefill(cfg, xBC, dtr, A, D, bias, conv_w=cw, conv_b=cb, z=z, norm_w=nw,
                         threads=1)
    pre = o.ssd_prefill(dict(cfg, seqlen=L0), xBC[:, :L0], dtr[:, :L0], A, D, bias, conv_w=cw,
                        conv_b=cb, z=z[:, :L0], norm_w=nw, threads=1)
    st = pre["h_final"].copy()
    cache = pre["conv_state_out"]
    worst = 0.0
    for j in range(k):
        t = L0 + j
        d = o.decode_step(dict(cfg, seqlen=1), xBC[:, t], dtr[:, t], A, D, bias, cw, cb, cache, st,
                          z_t=z[:, t], norm_w=nw)
        cache = d["conv_state_out"]
        worst = max(worst, _rel(d["out"], full["out"][:, t]))
    worst = max(worst, _rel(st, full["h_final"]))
    exact = np.array_equal(cache, xBC[:, -W:])
    return worst < 1e-12 and exact, f"rel err {worst:.2e} cache exact={exact}"


def pin_conv_impulse(o, seed=8):
    """P8: an impulse at t0 returns silu of the weights in reverse order; W = 1, w = 1 is silu."""
    r = _rng(seed)
    L, C, W, t0 = 12, 3, 4, 5
    xin = np.zeros((1, L, C))
    xin[0, t0, 1] = 1.0
    w = r.standard_normal((C, W))
    u = o.conv1d_silu(xin, w)
    ok = True
    for t in range(L):
        k = (W - 1) - (t - t0)
        want = o.silu(w[1, k]) if 0 <= k < W else 0.0
        ok = ok and abs(u[0, t, 1] - want) < 1e-15 and u[0, t, 0] == 0.0
    x2 = r.standard_normal((2, L, C))
    u2 = o.conv1d_silu(x2, np.ones((C, 1)))
    ok = ok and all(abs(u2[i] - o.silu(v)) < 1e-15 for i, v in np.ndenumerate(x2))
    return ok, ""


def pin_norm_invariants(o, seed=9):
    """P9: with eps = 0 and unit weights each group of the output has RMS exactly 1; the
    output is invariant to scaling g; groups are independent; z = 0 gates to 0; the plain
    RMSNorm gives unit RMS rows and scales with its weight."""
    r = _rng(seed)
    T, Dn, ng = 7, 24, 4
    y = r.standard_normal((T, Dn))
    z = r.standard_normal((T, Dn)) + 2.0
    out = o.gated_rmsnorm(y, z, None, ng, eps=0.0)
    rms = np.sqrt(np.mean(out.reshape(T, ng, -1) ** 2, axis=-1))
    ok = np.allclose(rms, 1.0, rtol=1e-14, atol=0)
    out2 = o.gated_rmsnorm(3.5 * y, z, None, ng, eps=0.0)
    ok = ok and np.allclose(out2, out, rtol=1e-13, atol=1e-15)
    y3 = y.copy()
    y3[:, :Dn // ng] *= 1000.0
    out3 = o.gated_rmsnorm(y3, z, None, ng, eps=0.0)
    ok = ok and np.allclose(out3[:, Dn // ng:], out[:, Dn // ng:], rtol=1e-13, atol=1e-15)
    outz = o.gated_rmsnorm(y, np.zeros((T, Dn)), None, ng, eps=1e-5)
    ok = ok and np.all(outz == 0.0)
    # the gate multiplies before normalising: a gate that is constant within a group cancels
    zc = np.repeat(r.uniform(1, 3, (T, ng)), Dn // ng, axis=1)
    ok = ok and np.allclose(o.gated_rmsnorm(y, zc, None, ng, eps=0.0),
                            o.gated_rmsnorm(y, None, None, ng, eps=0.0), rtol=1e-13, atol=1e-15)
    x = r.standard_normal((T, Dn))
    rn = o.rmsnorm(x, None, eps=0.0)
    ok = ok and np.allclose(np.sqrt(np.mean(rn ** 2, -1)), 1.0, rtol=1e-14, atol=0)
    wv = r.uniform(0.5, 2, Dn)
    ok = ok and np.allclose(o.rmsnorm(x, wv, eps=0.0), rn * wv, rtol=1e-14, atol=0)
    return bool(ok), ""


def pin_norm_before_gate(o, seed=13):
    """The normalise-first variant: with eps = 0 and unit weights, out / silu(z) has unit RMS
    in every group (the norm sees y alone); the gate is applied elementwise afterwards (a
    gate constant within a group does not cancel, unlike the gate-first form); without z both
    forms agree."""
    r = _rng(seed)
    T, Dn, ng = 6, 32, 4
    y = r.standard_normal((T, Dn))
    z = r.standard_normal((T, Dn)) + 2.0
    sz = z / (1.0 + np.exp(-z))
    out = o.gated_rmsnorm(y, z, None, ng, eps=0.0, norm_before_gate=True)
    rms = np.sqrt(np.mean((out / sz).reshape(T, ng, -1) ** 2, axis=-1))
    ok = np.allclose(rms, 1.0, rtol=1e-13, atol=0)
    plain = o.gated_rmsnorm(y, None, None, ng, eps=0.0)
    ok = ok and np.allclose(out, plain * sz, rtol=1e-13, atol=1e-15)
    ok = ok and np.allclose(o.gated_rmsnorm(y, None, None, ng, eps=0.0, norm_before_gate=True), plain,
                            rtol=1e-14, atol=0)
    zc = np.repeat(r.uniform(1, 3, (T, ng)), Dn // ng, axis=1)
    szc = zc / (1.0 + np.exp(-zc))
    ok = ok and np.allclose(o.gated_rmsnorm(y, zc, None, ng, eps=0.0, norm_before_gate=True), plain * szc,
                            rtol=1e-13, atol=1e-15)
    return bool(ok), ""


def pin_linearity(o, seed=10):
    """P10: with dt, B, C fixed and no conv, y and h_final are linear in (x, h0) jointly."""
    r = _rng(seed)
    B, L, H, G, P, N = 1, 17, 4, 2, 3, 4
    cfg = _raw_cfg(B, L, H, G, P, N)
    d = H * P
    base = r.standard_normal((B, L, d + 2 * G * N))
    x1, x2 = r.standard_normal((B, L, d)), r.standard_normal((B, L, d))
    h1, h2 = r.standard_normal((B, H, P, N)), r.standard_normal((B, H, P, N))
    dt = r.uniform(0.01, 0.3, (B, L, H))
    A, D = -r.uniform(1, 8, H), r.uniform(0, 1, H)
    al, be = 0.7, -1.9

    def run(x, h0):
        xb = base.copy()
        xb[..., :d] = x
        return o.ssd_prefill(cfg, xb, dt, A, D, np.zeros(H), h0=h0, threads=1)

    r1, r2, r3 = run(x1, h1), run(x2, h2), run(al * x1 + be * x2, al * h1 + be * h2)
    e = max(_rel(r3["y"], al * r1["y"] + be * r2["y"]),
            _rel(r3["h_final"], al * r1["h_final"] + be * r2["h_final"]))
    return e < 1e-12, f"rel err {e:.2e}"


def pin_mixer_composition(o, seed=11):
    """The mixer with identity projections is RMSNorm -> (z | xBC | dt) split -> scan+gated norm:
    W_in = I makes zxbcdt = rmsnorm(hidden); W_out = [I; 0] returns the gated output."""
    r = _rng(seed)
    B, L, H, G, P, N, W = 1, 9, 4, 2, 2, 3, 4
    d = H * P
    proj = 2 * d + 2 * G * N + H
    cfg = dict(_raw_cfg(B, L, H, G, P, N, W=W, softplus=True, dt_min=1e-3, dt_max=0.3,
                        norm_groups=2), d_model=proj, rms_eps=1e-5)
    hid = r.standard_normal((B, L, proj))
    bias, A, D = r.uniform(-4, -1, H), -r.uniform(1, 8, H), r.uniform(0, 1, H)
    cw = r.normal(0, 0.5, (d + 2 * G * N, W))
    nw = r.uniform(0.5, 1.5, d)
    W_out = np.zeros((proj, d))
    W_out[:d] = np.eye(d)
    out = o.mixer_forward(cfg, hid, None, np.eye(proj), W_out, A, D, bias, cw, None, nw,
                          bf16_activations=False)
    hn = o.rmsnorm(hid.reshape(-1, proj), None).reshape(B, L, proj)
    ref = o.ssd_prefill(cfg, np.ascontiguousarray(hn[..., d:2 * d + 2 * G * N]),
                        np.ascontiguousarray(hn[..., 2 * d + 2 * G * N:]), A, D, bias, conv_w=cw,
                        z=np.ascontiguousarray(hn[..., :d]), norm_w=nw, threads=1)
    e = _rel(out[..., :d], ref["out"])
    ok = e < 1e-12 and np.all(out[..., d:] == 0)
    return ok, f"rel err {e:.2e}"


def pin_bf16_rounding(o, seed=12):
    """Nearest-bf16 rounding: representable values are fixed points, ties go to the even
    mantissa, and on float32 inputs it agrees with the integer round-half-even of the bit
    pattern (an independent formulation); the vectorised form agrees with the scalar one."""
    from mamba_ssd_scan_02_b200 import datagen
    r = _rng(seed)
    cases = [(1.0, 1.0), (1.0 + 2 ** -8, 1.0), (1.0 + 3 * 2 ** -8, 1.0 + 2 ** -6),
             (-(1.0 + 2 ** -7), -(1.0 + 2 ** -7)), (1.0 + 2 ** -8 + 2 ** -30, 1.0 + 2 ** -7),
             (3.0e-3, float(datagen.bf16_value(datagen.bf16_bits(np.float32([3.0e-3])))[0])),
             (0.0, 0.0)]
    ok = all(o.round_bf16(x) == want for x, want in cases)
    x32 = (r.standard_normal(2000) * 10.0 ** r.uniform(-6, 6, 2000)).astype(np.float32)
    via_bits = datagen.bf16_value(datagen.bf16_bits(x32)).astype(np.float64)
    ok = ok and np.array_equal(o.round_bf16_array(x32.astype(np.float64)), via_bits)
    x64 = r.standard_normal(500) * 3.0
    ok = ok and np.array_equal(o._round_bf16_fast(x64), o.round_bf16_array(x64))
    return bool(ok), ""


ALL_PINS = [pin_activation_identities, pin_quadratic_form, pin_quadratic_with_conv,
            pin_prefix_sum, pin_zero_dt, pin_geometric, pin_chunk_invariance, pin_split_carry,
            pin_decode_equals_prefill, pin_conv_impulse, pin_norm_invariants, pin_linearity,
            pin_mixer_composition, pin_bf16_rounding, pin_norm_before_gate]

# planted mistakes in ssd_oracle.c (ORACLE_MUTANT values)
MUTANTS = {1: "D*x term dropped", 2: "sign of A flipped", 3: "output read before the update",
           4: "heads assigned to groups round-robin", 5: "conv taps reversed",
           6: "softplus skipped", 7: "B read in place of C"}
