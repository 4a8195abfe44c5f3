"""C-ABI checks that need no GPU: the library loads, exports every declared symbol, and
rejects invalid arguments on the host before anything is launched."""
import ctypes
import math
import os
import re

import pytest

from mamba_ssd_scan_02_b200 import ssd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssd.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"typedef\s+struct\s*\{.*?\}\s*\w+\s*;", "", text, flags=re.S)
    text = re.sub(r"typedef\s+enum\s*\{.*?\}\s*\w+\s*;", "", text, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\([^;]*\)\s*;", text, flags=re.M)


@pytest.fixture(scope="module")
def lib():
    return ssd.load()


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert set(names) >= {"ssd_prefill", "ssd_decode_step", "mamba2_mixer_forward"}
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ssd.h but not exported"
    assert set(ssd.EXPORTS) <= set(names)


def test_debug_build_exports_the_same_symbols(lib):
    """The normal build reports no index checks; the debug build (device-side index checks)
    exports every declared symbol too and reports its checks."""
    assert lib.ssd_debug_bounds_build() == 0
    if not os.path.exists(ssd.DEBUG_LIB_PATH):
        pytest.skip("libssd_debug.so not built")
    dbg = ctypes.CDLL(ssd.DEBUG_LIB_PATH)
    for n in declared_functions():
        assert hasattr(dbg, n), f"{n} not exported by the debug build"
    dbg.ssd_debug_bounds_build.restype = ctypes.c_int
    assert dbg.ssd_debug_bounds_build() == 1


def test_c_struct_layout_matches_header(lib):
    # sizes the header implies on LP64: 16 four-byte fields; pointer/long long fields are 8 bytes
    assert ctypes.sizeof(ssd.SsdConfig) == 17 * 4
    assert ctypes.sizeof(ssd.PrefillArgs) == 20 * 8
    assert ctypes.sizeof(ssd.DecodeArgs) == 17 * 8
    assert ctypes.sizeof(ssd.MixerArgs) == 17 * 8


def test_status_strings_and_version(lib):
    for code, name in ssd.STATUS.items():
        assert lib.ssd_status_string(code).decode().startswith(name)
    assert lib.ssd_version() >= 100


def _cfg(**kw):
    base = dict(batch=1, seqlen=256, nheads=8, ngroups=1, chunk=64, conv_width=4, dtype="bf16")
    base.update(kw)
    return ssd.make_config(base)


def _call_prefill(lib, c, **ptrs):
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: validation fails first
    a = ssd.PrefillArgs(xBC=fake, xBC_row_stride=8 * 64 + 256, dt=fake, dt_row_stride=8, A=fake,
                        D=fake, dt_bias=fake, conv_w=fake, y=fake, y_row_stride=8 * 64)
    for k, v in ptrs.items():
        setattr(a, k, v)
    return lib.ssd_prefill(ctypes.byref(c), ctypes.byref(a), None)


@pytest.mark.parametrize("kw,status", [
    (dict(headdim=32), 2), (dict(dstate=64), 2), (dict(chunk=96), 2), (dict(nheads=6, ngroups=4), 1),
    (dict(conv_width=5), 2), (dict(norm_groups=3), 1), (dict(batch=0), 1), (dict(seqlen=-1), 1),
])
def test_invalid_config_rejected(lib, kw, status):
    base = dict(batch=1, seqlen=256, nheads=8, ngroups=1, chunk=64, conv_width=4, dtype="bf16")
    base.update(kw)
    c = ssd.make_config(base)
    if "headdim" in kw:
        c.headdim = kw["headdim"]
    if "dstate" in kw:
        c.dstate = kw["dstate"]
    assert _call_prefill(lib, c) == status
    assert lib.ssd_workspace_size(ctypes.byref(c)) == 0


def test_invalid_pointers_rejected(lib):
    c = _cfg()
    assert _call_prefill(lib, c, xBC=None) == 1
    assert _call_prefill(lib, c, conv_w=None) == 1
    assert _call_prefill(lib, c, xBC=ctypes.c_void_p((1 << 20) + 2)) == 3  # misaligned
    assert _call_prefill(lib, c, y_row_stride=8 * 64 + 4) == 3             # stride not multiple of 8
    assert _call_prefill(lib, c, xBC_row_stride=100) == 1                   # stride < conv_dim
    # norm requested without z
    c2 = _cfg(norm_groups=1)
    assert _call_prefill(lib, c2) == 1
    # conv caches overlapping
    assert _call_prefill(lib, c, conv_state_in=ctypes.c_void_p(1 << 24),
                         conv_state_out=ctypes.c_void_p((1 << 24) + 64)) == 1
    # workspace missing
    assert _call_prefill(lib, c) == 7
    assert ssd.SsdConfig  # binding types exist
    assert lib.ssd_prefill(None, None, None) == 1


def test_workspace_size_grows_with_tokens(lib):
    a = lib.ssd_workspace_size(ctypes.byref(_cfg(seqlen=256)))
    b = lib.ssd_workspace_size(ctypes.byref(_cfg(seqlen=4096)))
    assert 0 < a < b and a % 256 == 0


def test_decode_rejects_bad_args(lib):
    c = _cfg(norm_groups=3, nheads=8, ngroups=2)
    fake = ctypes.c_void_p(1 << 20)
    a = ssd.DecodeArgs(xBC=fake, xBC_row_stride=8 * 64 + 512, dt=fake, dt_row_stride=8, A=fake,
                       D=fake, dt_bias=fake, conv_w=fake, state=fake, conv_state_in=fake,
                       conv_state_out=ctypes.c_void_p(1 << 26), y=fake, y_row_stride=512, z=fake,
                       z_row_stride=512)
    assert lib.ssd_decode_step(ctypes.byref(c), ctypes.byref(a), None) == 1   # 512 % 3 != 0
    c = _cfg(norm_groups=1, nheads=8, ngroups=2)
    assert lib.ssd_decode_step(ctypes.byref(c), ctypes.byref(a), None) == 2   # norm group spans groups
    c = _cfg(nheads=8, ngroups=2)
    a.state = None
    assert lib.ssd_decode_step(ctypes.byref(c), ctypes.byref(a), None) == 1


def test_mixer_rejects_bad_args(lib):
    m = ssd.MixerConfig(ssd=_cfg(), d_model=100, rms_eps=1e-5)
    a = ssd.MixerArgs()
    assert lib.mamba2_mixer_forward(ctypes.byref(m), ctypes.byref(a), None) == 2  # d_model % 64
    m.d_model = 512
    assert lib.mamba2_mixer_forward(ctypes.byref(m), ctypes.byref(a), None) == 1  # null pointers
    m.ssd.io_dtype = ssd.SSD_F32
    assert lib.mamba2_mixer_forward(ctypes.byref(m), ctypes.byref(a), None) == 2  # bf16 only
    assert lib.ssd_mixer_workspace_size(ctypes.byref(ssd.MixerConfig(ssd=_cfg(), d_model=512))) > 0
    assert not math.isnan(m.rms_eps)


def test_varlen_rejects_inconsistent_offsets(lib):
    """Checked on the host before anything is launched (no GPU needed)."""
    import ctypes
    from mamba_ssd_scan_02_b200 import ssd
    from mamba_ssd_scan_02_b200 import datagen
    cfg = dict(datagen.config(1), batch=1, seqlen=10)
    c = ssd.make_config(cfg)
    a = ssd.PrefillArgs()
    for cu in ([0, 6, 4, 10], [1, 5, 10], [0, 5, 9]):  # decreasing / not from 0 / wrong total
        arr = (ctypes.c_int * len(cu))(*cu)
        assert lib.ssd_prefill_varlen(ctypes.byref(c), ctypes.byref(a), arr, len(cu) - 1, None) == 1
        assert lib.ssd_varlen_workspace_size(ctypes.byref(c), arr, len(cu) - 1) == 0
    c2 = ssd.make_config(dict(cfg, batch=2))
    arr = (ctypes.c_int * 3)(0, 4, 10)
    assert lib.ssd_prefill_varlen(ctypes.byref(c2), ctypes.byref(a), arr, 2, None) == 1
