"""The C ABI of libfa_b200.so without a GPU: every symbol include/fa.h
declares is exported, and argument errors come back as status codes before
anything touches a device."""

import ctypes
import os
import re

import pytest

from exact_io_aware_bwd_b200 import binding
from exact_io_aware_bwd_b200.build import INCLUDE, build

HEADER = os.path.join(INCLUDE, "fa.h")


@pytest.fixture(scope="module")
def lib():
    build()
    return binding.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z_0-9]*\s*\**\s+\**\s*(fa_[a-z_0-9]+)\s*\(",
                       text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("fa_fwd", "fa_bwd", "fa_bwd_workspace_bytes", "fa_get_device_status",
              "fa_status_string"):
        assert n in names, names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in fa.h but not exported"


def test_status_strings(lib):
    for s in range(6):
        assert binding.fa_status_string(s)
    assert "unknown" in binding.fa_status_string(99)


FAKE = 1 << 20  # a 16-byte-aligned non-null pointer value; never dereferenced


def fwd_raw(lib, B=1, Hq=2, Hkv=2, N=128, d=64, scale=0.125, causal=0, dtype=0, ptrs=None):
    p = ptrs or [FAKE] * 5
    return lib.fa_fwd(*[ctypes.c_void_p(x) for x in p], B, Hq, Hkv, N, d, scale, causal, dtype, None)


def bwd_raw(lib, B=1, Hq=2, Hkv=2, N=128, d=64, scale=0.125, causal=0, dtype=0, ptrs=None,
            ws_bytes=None):
    p = ptrs or [FAKE] * 10
    ws = binding.fa_bwd_workspace_bytes(B, Hq, Hkv, N, d) if ws_bytes is None else ws_bytes
    vp = [ctypes.c_void_p(x) for x in p]
    return lib.fa_bwd(*vp[:9], B, Hq, Hkv, N, d, scale, causal, dtype, vp[9], ws, None)


@pytest.mark.parametrize("kw,status", [
    (dict(Hq=3, Hkv=2), binding.FA_ERR_INVALID_ARG),
    (dict(Hq=0), binding.FA_ERR_INVALID_ARG),
    (dict(Hkv=0), binding.FA_ERR_INVALID_ARG),
    (dict(B=-1), binding.FA_ERR_INVALID_ARG),
    (dict(N=-5), binding.FA_ERR_INVALID_ARG),
    (dict(scale=0.0), binding.FA_ERR_INVALID_ARG),
    (dict(scale=-1.0), binding.FA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), binding.FA_ERR_INVALID_ARG),
    (dict(scale=float("inf")), binding.FA_ERR_INVALID_ARG),
    (dict(causal=2), binding.FA_ERR_INVALID_ARG),
    (dict(d=96), binding.FA_ERR_UNSUPPORTED),
    (dict(d=256), binding.FA_ERR_UNSUPPORTED),
    (dict(dtype=7), binding.FA_ERR_UNSUPPORTED),
    (dict(ptrs=[FAKE, 0, FAKE, FAKE, FAKE]), binding.FA_ERR_INVALID_ARG),
    (dict(ptrs=[FAKE, FAKE + 8, FAKE, FAKE, FAKE]), binding.FA_ERR_MISALIGNED),
])
def test_fwd_argument_errors(lib, kw, status):
    assert fwd_raw(lib, **kw) == status


@pytest.mark.parametrize("kw,status", [
    (dict(Hq=4, Hkv=3), binding.FA_ERR_INVALID_ARG),
    (dict(d=32), binding.FA_ERR_UNSUPPORTED),
    (dict(ws_bytes=100), binding.FA_ERR_INVALID_ARG),
    (dict(ptrs=[FAKE] * 9 + [0]), binding.FA_ERR_INVALID_ARG),
    (dict(ptrs=[FAKE] * 6 + [FAKE + 4] + [FAKE] * 3), binding.FA_ERR_MISALIGNED),
])
def test_bwd_argument_errors(lib, kw, status):
    assert bwd_raw(lib, **kw) == status


def test_empty_problems_are_no_ops(lib):
    # B == 0 or N == 0: nothing to compute, nothing launched, even with null pointers
    assert fwd_raw(lib, B=0, ptrs=[0] * 5) == binding.FA_OK
    assert fwd_raw(lib, N=0, ptrs=[0] * 5) == binding.FA_OK
    assert bwd_raw(lib, N=0, ptrs=[0] * 10, ws_bytes=0) == binding.FA_OK
    assert binding.fa_bwd_workspace_bytes(1, 2, 2, 0, 64) == 0


def test_workspace_is_linear_in_n():
    # two fp32 row statistics + an fp32 dQ accumulator per (padded) query row,
    # plus a fixed 256-byte tail (the main pass's work-item counter)
    tail = 256
    for d in (64, 128):
        sizes = [binding.fa_bwd_workspace_bytes(1, 16, 16, n, d) - tail
                 for n in (4096, 8192, 16384, 32768, 65536)]
        for a, b in zip(sizes, sizes[1:]):
            assert b == 2 * a
        assert sizes[0] == 16 * 4096 * 4 * (2 + d)
    # padding to a multiple of 128 rows
    assert binding.fa_bwd_workspace_bytes(1, 1, 1, 129, 64) == 256 * 4 * 66 + tail


def test_blockmask_workspace_and_argument_errors(lib):
    vp = ctypes.c_void_p
    B, Hq, Hkv, N, d = 2, 8, 2, 1000, 128
    nb = -(-N // 128)
    plain = binding.fa_bwd_workspace_bytes(B, Hq, Hkv, N, d)
    # per work item (kv head x key block): a step count and a walk of at most
    # group x nb two-byte entries
    assert binding.fa_bwd_blockmask_workspace_bytes(B, Hq, Hkv, N, d) == \
        plain + 4 * B * Hkv * nb + 2 * B * Hkv * nb * (Hq // Hkv) * nb
    assert binding.fa_bwd_blockmask_workspace_bytes(1, 3, 2, 256, 64) == 0  # Hq % Hkv
    fwd = lambda mask, per_head, Hq=2, Hkv=2, N=256: lib.fa_fwd_blockmask(
        *([vp(FAKE)] * 5 + [1, Hq, Hkv, N, 64, 0.125, 1, mask, per_head, binding.FA_BF16, None]))
    assert fwd(None, 0) == binding.FA_ERR_INVALID_ARG                 # no mask
    assert fwd(vp(FAKE), 2) == binding.FA_ERR_INVALID_ARG             # per_head not 0/1
    assert fwd(vp(FAKE), 0, Hq=34, Hkv=2) == binding.FA_ERR_UNSUPPORTED  # group > 16
    assert fwd(vp(FAKE), 0, N=4096 * 128 + 1) == binding.FA_ERR_UNSUPPORTED  # nb > 4096
    ws = binding.fa_bwd_blockmask_workspace_bytes(1, 2, 2, 256, 64)
    bwd = lambda mask, per_head, ws_bytes=ws: lib.fa_bwd_blockmask(
        *([vp(FAKE)] * 9 + [1, 2, 2, 256, 64, 0.125, 1, mask, per_head, binding.FA_BF16, vp(FAKE),
                            ws_bytes, None]))
    assert bwd(None, 1) == binding.FA_ERR_INVALID_ARG
    assert bwd(vp(FAKE), 1, binding.fa_bwd_workspace_bytes(1, 2, 2, 256, 64)) == binding.FA_ERR_INVALID_ARG
    # empty problems are no-ops
    assert lib.fa_fwd_blockmask(*([vp(0)] * 5 + [0, 2, 2, 256, 64, 0.125, 1, vp(FAKE), 0,
                                                 binding.FA_BF16, None])) == binding.FA_OK


def test_bwd_max_blocks_setting(lib):
    assert lib.fa_set_bwd_max_blocks(-1) == binding.FA_ERR_INVALID_ARG
    assert lib.fa_set_bwd_max_blocks(3) == binding.FA_OK
    assert lib.fa_set_bwd_max_blocks(0) == binding.FA_OK


def test_window_entry_points_check_their_arguments(lib):
    vp = ctypes.c_void_p
    args = lambda w: [vp(FAKE)] * 5 + [1, 2, 2, 256, 64, 0.125, w, binding.FA_BF16, None]
    assert lib.fa_fwd_window(*args(0)) == binding.FA_ERR_INVALID_ARG
    assert lib.fa_fwd_window(*args(-3)) == binding.FA_ERR_INVALID_ARG
    ws = binding.fa_bwd_workspace_bytes(1, 2, 2, 256, 64)
    bargs = lambda w, d=64: ([vp(FAKE)] * 9 + [1, 2, 2, 256, d, 0.125, w, binding.FA_BF16,
                                               vp(FAKE), ws, None])
    assert lib.fa_bwd_window(*bargs(0)) == binding.FA_ERR_INVALID_ARG
    assert lib.fa_bwd_window(*bargs(16, d=96)) == binding.FA_ERR_UNSUPPORTED
    # empty problems are no-ops here too
    assert lib.fa_fwd_window(*([vp(0)] * 5 + [0, 2, 2, 256, 64, 0.125, 8, binding.FA_BF16, None])) == binding.FA_OK


@pytest.mark.parametrize("p_drop", [-0.1, 1.0, 0.999, float("nan"), float("inf")])
def test_dropout_entry_points_reject_bad_rates(lib, p_drop):
    vp = ctypes.c_void_p
    args = [vp(FAKE)] * 5 + [1, 2, 2, 256, 64, 0.125, 1, p_drop, 7, binding.FA_BF16, None]
    assert lib.fa_fwd_dropout(*args) == binding.FA_ERR_INVALID_ARG
    ws = binding.fa_bwd_workspace_bytes(1, 2, 2, 256, 64)
    bargs = [vp(FAKE)] * 9 + [1, 2, 2, 256, 64, 0.125, 1, p_drop, 7, binding.FA_BF16, vp(FAKE), ws, None]
    assert lib.fa_bwd_dropout(*bargs) == binding.FA_ERR_INVALID_ARG


def test_dropout_entry_points_accept_good_rates_on_empty_problems(lib):
    vp = ctypes.c_void_p
    for p_drop in (0.0, 0.1, 0.5, 0.99):
        args = [vp(0)] * 5 + [0, 2, 2, 256, 64, 0.125, 1, p_drop, 7, binding.FA_BF16, None]
        assert lib.fa_fwd_dropout(*args) == binding.FA_OK


def test_fp8_forward_argument_errors(lib):
    vp = ctypes.c_void_p

    def call(B=1, Hq=2, Hkv=2, N=256, d=128, scale=0.09, ds=(0.01, 0.02, 0.03), causal=1,
             dtype=binding.FA_BF16, ptrs=None):
        p = ptrs if ptrs is not None else [FAKE] * 5
        return lib.fa_fwd_fp8(*[vp(x) for x in p], B, Hq, Hkv, N, d, scale, *ds, causal, dtype, None)

    for bad in (0.0, -1.0, float("nan"), float("inf")):
        for i in range(3):
            ds = [0.01, 0.02, 0.03]
            ds[i] = bad
            assert call(ds=tuple(ds)) == binding.FA_ERR_INVALID_ARG, (i, bad)
    assert call(ds=(1e30, 1e30, 1.0)) == binding.FA_ERR_INVALID_ARG   # scale * factors overflows
    assert call(d=64) == binding.FA_ERR_UNSUPPORTED
    assert call(dtype=7) == binding.FA_ERR_UNSUPPORTED
    assert call(Hq=3) == binding.FA_ERR_INVALID_ARG
    assert call(causal=2) == binding.FA_ERR_INVALID_ARG
    assert call(ptrs=[FAKE] * 4 + [0]) == binding.FA_ERR_INVALID_ARG
    assert call(ptrs=[FAKE + 8] + [FAKE] * 4) == binding.FA_ERR_MISALIGNED
    assert call(B=0, ptrs=[0] * 5) == binding.FA_OK
    assert call(N=0, ptrs=[0] * 5) == binding.FA_OK


def test_decode_argument_errors(lib):
    vp = ctypes.c_void_p
    ws = binding.fa_decode_workspace_bytes(2, 8, 2, 1, 128, 16)
    assert ws > 0

    def call(B=2, Hq=8, Hkv=2, Nq=1, d=128, P=64, max_pages=16, num_pages=40, scale=0.1,
             dtype=binding.FA_BF16, ptrs=None, ws_bytes=ws):
        p = ptrs if ptrs is not None else [FAKE] * 7
        return lib.fa_decode_paged(*[vp(x) for x in p], B, Hq, Hkv, Nq, d, P, max_pages, num_pages,
                                   scale, dtype, vp(FAKE), ws_bytes, None)

    assert call(Hq=7) == binding.FA_ERR_INVALID_ARG
    assert call(Nq=0) == binding.FA_ERR_INVALID_ARG
    assert call(max_pages=0) == binding.FA_ERR_INVALID_ARG
    assert call(scale=0.0) == binding.FA_ERR_INVALID_ARG
    assert call(d=96) == binding.FA_ERR_UNSUPPORTED
    assert call(P=48) == binding.FA_ERR_UNSUPPORTED
    assert call(Hq=16, Hkv=1, Nq=4) == binding.FA_ERR_UNSUPPORTED      # 64 rows per kv head
    assert call(ws_bytes=ws - 4) == binding.FA_ERR_INVALID_ARG
    assert call(ptrs=[FAKE] * 6 + [0]) == binding.FA_ERR_INVALID_ARG
    assert call(ptrs=[FAKE + 8] + [FAKE] * 6) == binding.FA_ERR_MISALIGNED
    assert call(B=0, ptrs=[0] * 7) == binding.FA_OK


def test_missing_library_fails_loudly(tmp_path):
    """No fallback: with the library absent the binding raises instead of
    computing anything another way."""
    import subprocess
    import sys
    code = ("import sys; sys.path.insert(0, %r)\n"
            "from exact_io_aware_bwd_b200 import binding\n"
            "try:\n    binding.load()\nexcept RuntimeError as e:\n    print('raised', e)\n"
            % os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    env = dict(os.environ, FA_B200_LIB=str(tmp_path / "absent.so"))
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert "raised" in r.stdout and "no fallback" in r.stdout
