"""Host-side checks of the C-ABI library (no GPU needed): it loads, exports every entry point
include/rtp.h declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for f in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if f.endswith(".h"):
            text = open(os.path.join(ROOT, "include", f)).read()
            names += re.findall(r"^RTP_API\s+[\w\s\*]*?\b(rtp_\w+)\s*\(", text, re.M)
    return names


def test_header_declares_entry_points():
    names = _declared()
    assert "rtp_create" in names and "rtp_decode_step" in names and "rtp_destroy" in names
    assert len(names) == len(set(names))


def test_library_exports_every_declared_symbol(rtp_lib):
    lib = rtp_lib.load()
    for name in _declared():
        assert hasattr(lib, name), f"librtp.so does not export {name}"
    assert set(_declared()) == set(rtp_lib.EXPORTS)


def test_config_default_matches_pages(rtp_lib):
    c = rtp_lib.default_config(48, 1, 32, 4, 1 << 20)
    assert (c.head_dim, c.idx_dim, c.window, c.sinks, c.num_bins) == (128, 16, 8192, 4, 256)
    assert c.idx_range == 16.0 and c.idx_scale == 0.25
    assert abs(c.attn_scale - 128 ** -0.5) < 1e-7


def test_workspace_is_linear_in_context(rtp_lib):
    a = rtp_lib.workspace_bytes(rtp_lib.default_config(1, 1, 32, 4, 1 << 18))
    b = rtp_lib.workspace_bytes(rtp_lib.default_config(1, 1, 32, 4, 1 << 20))
    c = rtp_lib.workspace_bytes(rtp_lib.default_config(1, 1, 32, 4, 1 << 21))
    # linear in max_ctx: b - a covers 3 * 2^18 more tokens, c - b covers 4 * 2^18
    assert 0 < a < b < c and abs(3 * (c - b) - 4 * (b - a)) < 0.05 * (c - b)
    assert rtp_lib.workspace_bytes(rtp_lib.default_config(1, 1, 32, 4, 0)) == 0


@pytest.mark.parametrize("field,value,status", [
    ("head_dim", 64, 2), ("idx_dim", 32, 2), ("num_bins", 128, 2), ("num_q_heads", 36, 2),
    ("num_q_heads", 30, 1), ("max_ctx", 0, 1), ("window", 0, 1), ("sinks", -1, 1),
    ("idx_range", 0.0, 1), ("idx_scale", -1.0, 1), ("attn_scale", float("inf"), 1),
    ("batch", 0, 1), ("num_layers", 0, 1), ("max_ctx", 1 << 24, 1), ("max_ctx", 1 << 28, 1),
])
def test_create_rejects_bad_config_before_touching_the_device(rtp_lib, field, value, status):
    c = rtp_lib.default_config(2, 1, 32, 4, 4096)
    setattr(c, field, value)
    h = ctypes.c_void_p()
    st = rtp_lib.load().rtp_create(ctypes.byref(c), 0, ctypes.byref(h))
    assert st == status
    assert not h.value
    assert rtp_lib.load().rtp_last_error().decode()


def test_max_ctx_stops_where_the_fixed_point_mass_sums_would_wrap(rtp_lib):
    """Token masses in (0, 1] are summed as 64-bit integers of 2^-40 units: N tokens of mass 1
    reach N * 2^40, which wraps at N = 2^24. The last context that cannot wrap is accepted, the
    first one that can is refused."""
    ok = rtp_lib.workspace_bytes(rtp_lib.default_config(1, 1, 8, 1, (1 << 24) - 1))
    assert ok > 0
    assert ((1 << 24) - 1) * (1 << 40) < 1 << 64 <= (1 << 24) * (1 << 40)
    assert rtp_lib.workspace_bytes(rtp_lib.default_config(1, 1, 8, 1, 1 << 24)) == 0
    c = rtp_lib.default_config(1, 1, 8, 1, 1 << 24)
    h = ctypes.c_void_p()
    assert rtp_lib.load().rtp_create(ctypes.byref(c), 0, ctypes.byref(h)) == \
        rtp_lib.RTP_ERR_INVALID_ARG
    assert "2^24" in rtp_lib.load().rtp_last_error().decode()


def test_calls_on_null_handle_are_rejected(rtp_lib):
    L = rtp_lib.load()
    io = rtp_lib.LayerIO()
    assert L.rtp_decode_step(None, 0, ctypes.byref(io), None) == rtp_lib.RTP_ERR_INVALID_ARG
    assert L.rtp_dense_decode(None, ctypes.byref(io), None) == rtp_lib.RTP_ERR_INVALID_ARG
    cnt = ctypes.c_int64()
    assert L.rtp_get_selection(None, 0, 0, None, 0, ctypes.byref(cnt)) == 1
    assert L.rtp_selftest_wait_timeout(None, 0, ctypes.byref(io), 1000000, None) == \
        rtp_lib.RTP_ERR_INVALID_ARG
    assert L.rtp_nvtx_enable(None, 1) == rtp_lib.RTP_ERR_INVALID_ARG
    n = ctypes.c_int64()
    assert L.rtp_profile_launches(None, None, None, 0, ctypes.byref(n)) == \
        rtp_lib.RTP_ERR_INVALID_ARG
    pio = rtp_lib.PrefillIO()
    assert L.rtp_prefill(None, ctypes.byref(pio), None) == rtp_lib.RTP_ERR_INVALID_ARG
    assert L.rtp_destroy(None) == rtp_lib.RTP_OK
    assert L.rtp_status_string(3) == b"RTP_ERR_OOM"


def test_workspace_holds_single_launch_buffers_only_within_its_limits(rtp_lib):
    """The single-launch layer's pieces (one per CTA and head, 4160 bytes each), masks and keys
    are planned for B * Hkv <= 64 only: 68 heads need less workspace than 64."""
    ws = lambda B: rtp_lib.workspace_bytes(rtp_lib.default_config(1, B, 32, 4, 4096))
    within, beyond = ws(16), ws(17)          # 64 heads, then 68 heads
    assert 0 < beyond < within
    assert within - beyond > 16 << 20        # 64 x (one piece per SM) x 4160 B alone is ~39 MB


@pytest.mark.parametrize("compiler,std,lang", [("gcc", "-std=c99", "c"), ("g++", "-std=c++17", "c++")])
def test_header_compiles_as_c_and_cpp(tmp_path, compiler, std, lang):
    """include/rtp.h is a plain C header (no torch, no CUDA types in the signatures)."""
    import shutil
    import subprocess
    if shutil.which(compiler) is None:
        pytest.skip(f"{compiler} not installed")
    src = tmp_path / "use_rtp.c"
    src.write_text('#include "rtp.h"\nint main(void) { rtp_layer_io io; io.single_launch = 1;'
                   ' (void)io; return rtp_status_string(RTP_OK) ? 0 : 1; }\n')
    r = subprocess.run([compiler, std, "-Wall", "-Wextra", "-Werror", "-fsyntax-only", "-x", lang,
                        "-I", os.path.join(ROOT, "include"), str(src)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
