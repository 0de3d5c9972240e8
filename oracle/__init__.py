"""CPU oracle for exact softmax attention (forward and backward) in fp64.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package.  It shares no
code with the GPU library (no common kernels, headers, helpers or constants)
and never imports it.

The arithmetic lives in ``oracle.c`` (plain C, fp64, one thread per
independent head); this module compiles it with gcc on first use and wraps
it for numpy arrays.  Every function follows the plain definition of
attention given on the pages ("flash attention io aware", section "The
Memory Bandwidth Bottleneck": S = QK^T, P = softmax(S), O = PV),
with the softmax statistics kept as one natural-log logsumexp per row
("FlashAttention" glossary, recomputation paragraph: the backward pass keeps
only the normalisation statistics).  The backward formulas are the calculus
of softmax; ``oracle.c`` writes them out in its header.

Parity status of each function (what pins it, see tests/test_oracle_pins.py):
  fwd, fwd_rows          closed forms (Q = 0, one-hot keys, causal row 0),
                         hand-derived golden values, torch fp64 SDPA,
                         brute-force Python loops
  fwd_online             equal to the two-pass form within 1e-12 (fp64)
  e4m3_decode            every code against torch.float8_e4m3fn, values
                         hand-derived from the format's definition
  fwd_fp8, fwd_fp8_rows  closed form at Q = 0, torch fp64 SDPA on the
                         dequantised values, moving a power of two between
                         the query and key factors changes nothing
  block_mask= (every     a mask of ones changes nothing, block-diagonal masks
  attention function)    split into independent problems, pure-Python loops,
                         torch fp64 SDPA + autograd with the expanded mask,
                         rows that see no block (O = 0, lse = -inf, no
                         gradient), row/column/online forms agree
  bwd, bwd_rows,         central finite differences of the forward,
  bwd_cols               closed forms at Q = 0, torch fp64 autograd,
                         gradient invariants, hand-derived golden values
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_default = None

_i64 = ctypes.c_int64
_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False, src: str = SOURCE, out: str = _LIB_PATH) -> str:
    """Compile ``src`` (default oracle.c) into the shared library ``out`` (gcc -O2, no fast-math)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", src, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, out)
    return out


def _f64(a) -> np.ndarray:
    """Exact upcast of an array (numpy or torch CPU tensor) to contiguous fp64."""
    if hasattr(a, "detach"):
        a = a.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(_dp)


def _codes(a) -> np.ndarray:
    """8-bit codes (numpy uint8, or a torch uint8 / float8 CPU tensor) as contiguous uint8."""
    if hasattr(a, "detach"):
        import torch
        a = a.detach().cpu()
        if a.dtype != torch.uint8:
            a = a.view(torch.uint8)
        a = a.numpy()
    a = np.asarray(a)
    if a.dtype != np.uint8:
        raise ValueError(f"expected 8-bit codes, got {a.dtype}")
    return np.ascontiguousarray(a)


def _dims(q, k):
    B, Hq, N, d = q.shape
    Bk, Hkv, Nk, dk = k.shape
    if (Bk, Nk, dk) != (B, N, d) or Hq % Hkv:
        raise ValueError(f"incompatible shapes q{q.shape} k{k.shape}")
    return B, Hq, Hkv, N, d


def _drop(dropout):
    """(drop_t, seed_lo, seed_hi) from dropout = None or (t, seed): t the 8-bit
    threshold (a key is dropped when its random byte is below t), seed 64-bit."""
    if not dropout:
        return 0, 0, 0
    t, seed = dropout
    seed = int(seed) & 0xFFFFFFFFFFFFFFFF
    return int(t), seed & 0xFFFFFFFF, seed >> 32


def _bmask(block_mask, Hq: int, N: int):
    """The C arguments (pointer, head stride, bq, bk) of block_mask = None or
    (mask, bq, bk): mask [Tq, Tk] shared by every head, or [Hq, Tq, Tk], with
    Tq = ceil(N / bq), Tk = ceil(N / bk); nonzero = the block is computed.
    Returns (array to keep alive, arguments)."""
    if block_mask is None:
        return None, (None, 0, 0, 0)
    mask, bq, bk = block_mask
    bq, bk = int(bq), int(bk)
    if bq <= 0 or bk <= 0:
        raise ValueError("block sizes must be positive")
    m = mask.detach().cpu().numpy() if hasattr(mask, "detach") else np.asarray(mask)
    m = np.ascontiguousarray(m != 0, dtype=np.uint8)
    Tq, Tk = -(-N // bq), -(-N // bk)
    if m.shape == (Tq, Tk):
        hstride = 0
    elif m.shape == (Hq, Tq, Tk):
        hstride = Tq * Tk
    else:
        raise ValueError(f"block mask of shape {m.shape}: expected ({Tq}, {Tk}) or ({Hq}, {Tq}, {Tk})")
    return m, (m.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)), hstride, bq, bk)


class Oracle:
    """numpy-facing wrapper of one compiled copy of the oracle library."""

    def __init__(self, lib_path: str):
        lib = ctypes.CDLL(lib_path)
        u32 = ctypes.c_uint32
        # B, Hq, Hkv, N, d, scale, causal, window, drop_t, seed_lo, seed_hi,
        # block mask, its head stride, block rows, block columns
        common = [_i64, _i64, _i64, _i64, _i64, ctypes.c_double, ctypes.c_int, _i64, ctypes.c_int, u32, u32,
                  ctypes.POINTER(ctypes.c_uint8), _i64, _i64, _i64]
        lib.oracle_fwd.argtypes = [_dp, _dp, _dp, _dp, _dp] + common + [ctypes.c_int]
        lib.oracle_fwd_rows.argtypes = [_dp, _dp, _dp, _ip, _i64, _dp, _dp] + common + [ctypes.c_int]
        lib.oracle_fwd_online.argtypes = [_dp, _dp, _dp, _dp, _dp] + common + [_i64, ctypes.c_int]
        lib.oracle_bwd.argtypes = [_dp, _dp, _dp, _dp, _dp, _dp, _dp] + common + [ctypes.c_int]
        lib.oracle_bwd_rows.argtypes = [_dp, _dp, _dp, _dp, _ip, _i64, _dp] + common + [ctypes.c_int]
        lib.oracle_bwd_cols.argtypes = ([_dp, _dp, _dp, _dp, _i64, _i64, _ip, _i64, _dp, _dp]
                                        + common + [ctypes.c_int])
        lib.oracle_num_threads.argtypes = [ctypes.c_int]
        lib.oracle_decode_paged.argtypes = ([_dp, _dp, _dp, _ip, _ip, _dp, _dp]
                                            + [_i64] * 8 + [ctypes.c_double, ctypes.c_int])
        lib.oracle_decode_paged.restype = ctypes.c_int
        lib.oracle_philox4x32_10.argtypes = [ctypes.POINTER(u32), ctypes.POINTER(u32), ctypes.POINTER(u32)]
        lib.oracle_philox4x32_10.restype = None
        lib.oracle_e4m3_decode.argtypes = [ctypes.POINTER(ctypes.c_uint8), _i64, _dp]
        lib.oracle_e4m3_decode.restype = None
        for f in ("oracle_fwd", "oracle_fwd_rows", "oracle_fwd_online", "oracle_bwd",
                  "oracle_bwd_rows", "oracle_bwd_cols", "oracle_num_threads"):
            getattr(lib, f).restype = ctypes.c_int
        self.lib = lib

    def philox4x32_10(self, ctr, key):
        """Philox4x32-10 of a 4-word counter and 2-word key: 4 words."""
        c = (ctypes.c_uint32 * 4)(*[int(x) & 0xFFFFFFFF for x in ctr])
        k = (ctypes.c_uint32 * 2)(*[int(x) & 0xFFFFFFFF for x in key])
        o = (ctypes.c_uint32 * 4)()
        self.lib.oracle_philox4x32_10(c, k, o)
        return [int(x) for x in o]

    def e4m3_decode(self, codes) -> np.ndarray:
        """The exact fp64 value of every E4M3 code (NaN for the NaN codes)."""
        c = _codes(codes)
        out = np.zeros(c.shape, dtype=np.float64)
        self.lib.oracle_e4m3_decode(c.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)), c.size, _ptr(out))
        return out

    def _dequant(self, q8, k8, v8, descale):
        dq, dk, dv = (float(x) for x in descale)
        return self.e4m3_decode(q8) * dq, self.e4m3_decode(k8) * dk, self.e4m3_decode(v8) * dv

    def fwd_fp8(self, q8, k8, v8, descale, scale: float, causal: bool, nthreads: int = 0):
        """O and lse of attention on E4M3 inputs: the definition applied to
        descale[0] * Q8, descale[1] * K8, descale[2] * V8 (exact in fp64)."""
        q, k, v = self._dequant(q8, k8, v8, descale)
        return self.fwd(q, k, v, scale, causal, nthreads)

    def fwd_fp8_rows(self, q8, k8, v8, descale, rows, scale: float, causal: bool, nthreads: int = 0):
        """``fwd_fp8`` for the query rows ``rows`` of every head."""
        q, k, v = self._dequant(q8, k8, v8, descale)
        return self.fwd_rows(q, k, v, rows, scale, causal, nthreads)

    def num_threads(self, nthreads: int = 0) -> int:
        """Threads the oracle uses for ``nthreads`` (<= 0: every online core)."""
        return self.lib.oracle_num_threads(nthreads)

    def fwd(self, q, k, v, scale: float, causal: bool, nthreads: int = 0, *, window: int = 0, dropout=None,
            block_mask=None):
        """O [B,Hq,N,d] and lse [B,Hq,N] (natural log), materialising N x N per head."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        B, Hq, Hkv, N, d = _dims(q, k)
        keep, margs = _bmask(block_mask, Hq, N)
        o = np.zeros((B, Hq, N, d))
        lse = np.zeros((B, Hq, N))
        rc = self.lib.oracle_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                 B, Hq, Hkv, N, d, float(scale), int(causal), int(window), *_drop(dropout),
                                 *margs, nthreads)
        if rc:
            raise ValueError(f"oracle_fwd rejected its arguments ({rc})")
        return o, lse

    def fwd_rows(self, q, k, v, rows, scale: float, causal: bool, nthreads: int = 0, *,
                 window: int = 0, dropout=None, block_mask=None):
        """O and lse of the query rows ``rows`` of every head: [B,Hq,R,d], [B,Hq,R]."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        B, Hq, Hkv, N, d = _dims(q, k)
        keep, margs = _bmask(block_mask, Hq, N)
        rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        R = rows.size
        o = np.zeros((B, Hq, R, d))
        lse = np.zeros((B, Hq, R))
        rc = self.lib.oracle_fwd_rows(_ptr(q), _ptr(k), _ptr(v), rows.ctypes.data_as(_ip), R,
                                      _ptr(o), _ptr(lse), B, Hq, Hkv, N, d, float(scale),
                                      int(causal), int(window), *_drop(dropout), *margs, nthreads)
        if rc:
            raise ValueError(f"oracle_fwd_rows rejected its arguments ({rc})")
        return o, lse

    def fwd_online(self, q, k, v, scale: float, causal: bool, block: int = 128, nthreads: int = 0,
                   *, window: int = 0, dropout=None, block_mask=None):
        """O and lse by the one-pass blocked online softmax (not the definition)."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        B, Hq, Hkv, N, d = _dims(q, k)
        keep, margs = _bmask(block_mask, Hq, N)
        o = np.zeros((B, Hq, N, d))
        lse = np.zeros((B, Hq, N))
        rc = self.lib.oracle_fwd_online(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                        B, Hq, Hkv, N, d, float(scale), int(causal), int(window), *_drop(dropout),
                                        *margs, int(block), nthreads)
        if rc:
            raise ValueError(f"oracle_fwd_online rejected its arguments ({rc})")
        return o, lse

    def bwd(self, q, k, v, dout, scale: float, causal: bool, nthreads: int = 0, *, window: int = 0, dropout=None,
            block_mask=None):
        """dQ [B,Hq,N,d], dK, dV [B,Hkv,N,d] (dK, dV summed over each query group)."""
        q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
        B, Hq, Hkv, N, d = _dims(q, k)
        keep, margs = _bmask(block_mask, Hq, N)
        dq = np.zeros((B, Hq, N, d))
        dk = np.zeros((B, Hkv, N, d))
        dv = np.zeros((B, Hkv, N, d))
        rc = self.lib.oracle_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq), _ptr(dk),
                                 _ptr(dv), B, Hq, Hkv, N, d, float(scale), int(causal), int(window), *_drop(dropout),
                                 *margs, nthreads)
        if rc:
            raise ValueError(f"oracle_bwd rejected its arguments ({rc})")
        return dq, dk, dv

    def bwd_rows(self, q, k, v, dout, rows, scale: float, causal: bool, nthreads: int = 0, *,
                 window: int = 0, dropout=None, block_mask=None):
        """dQ of the query rows ``rows`` of every head: [B,Hq,R,d]."""
        q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
        B, Hq, Hkv, N, d = _dims(q, k)
        keep, margs = _bmask(block_mask, Hq, N)
        rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        R = rows.size
        dq = np.zeros((B, Hq, R, d))
        rc = self.lib.oracle_bwd_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(dout),
                                      rows.ctypes.data_as(_ip), R, _ptr(dq),
                                      B, Hq, Hkv, N, d, float(scale), int(causal), int(window), *_drop(dropout),
                                      *margs, nthreads)
        if rc:
            raise ValueError(f"oracle_bwd_rows rejected its arguments ({rc})")
        return dq

    def bwd_cols(self, q, k, v, dout, b: int, hkv: int, cols, scale: float, causal: bool,
                 nthreads: int = 0, *, window: int = 0, dropout=None, block_mask=None):
        """dK and dV of key rows ``cols`` of kv head (b, hkv): [C,d] each."""
        q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
        B, Hq, Hkv, N, d = _dims(q, k)
        keep, margs = _bmask(block_mask, Hq, N)
        cols = np.ascontiguousarray(np.asarray(cols, dtype=np.int64))
        C = cols.size
        dk = np.zeros((C, d))
        dv = np.zeros((C, d))
        rc = self.lib.oracle_bwd_cols(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), int(b), int(hkv),
                                      cols.ctypes.data_as(_ip), C, _ptr(dk), _ptr(dv),
                                      B, Hq, Hkv, N, d, float(scale), int(causal), int(window), *_drop(dropout),
                                      *margs, nthreads)
        if rc:
            raise ValueError(f"oracle_bwd_cols rejected its arguments ({rc})")
        return dk, dv


    def decode_paged(self, q, k_cache, v_cache, block_table, seq_lens, scale: float,
                     nthreads: int = 0):
        """Decode over a paged cache: q [B,Hq,Nq,d], caches [pages,Hkv,P,d],
        block_table [B,max_pages], seq_lens [B] -> O [B,Hq,Nq,d], lse [B,Hq,Nq]."""
        q, kc, vc = _f64(q), _f64(k_cache), _f64(v_cache)
        B, Hq, Nq, d = q.shape
        num_pages, Hkv, P, dk = kc.shape
        if dk != d or vc.shape != kc.shape or Hq % Hkv:
            raise ValueError("incompatible shapes")
        table = np.ascontiguousarray(np.asarray(block_table, dtype=np.int64).reshape(B, -1))
        lens = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int64).reshape(B))
        o = np.zeros((B, Hq, Nq, d))
        lse = np.zeros((B, Hq, Nq))
        rc = self.lib.oracle_decode_paged(_ptr(q), _ptr(kc), _ptr(vc), table.ctypes.data_as(_ip),
                                          lens.ctypes.data_as(_ip), _ptr(o), _ptr(lse), B, Hq, Hkv,
                                          Nq, d, P, table.shape[1], num_pages, float(scale), nthreads)
        if rc:
            raise ValueError(f"oracle_decode_paged rejected its arguments ({rc})")
        return o, lse


def default() -> Oracle:
    """The oracle compiled from oracle.c (built on first use)."""
    global _default
    with _lock:
        if _default is None:
            _default = Oracle(build())
    return _default


def num_threads(nthreads: int = 0) -> int:
    return default().num_threads(nthreads)


def fwd(*a, **kw):
    return default().fwd(*a, **kw)


def fwd_rows(*a, **kw):
    return default().fwd_rows(*a, **kw)


def fwd_online(*a, **kw):
    return default().fwd_online(*a, **kw)


def bwd(*a, **kw):
    return default().bwd(*a, **kw)


def bwd_rows(*a, **kw):
    return default().bwd_rows(*a, **kw)


def bwd_cols(*a, **kw):
    return default().bwd_cols(*a, **kw)


def decode_paged(*a, **kw):
    return default().decode_paged(*a, **kw)


def e4m3_decode(*a, **kw):
    return default().e4m3_decode(*a, **kw)


def fwd_fp8(*a, **kw):
    return default().fwd_fp8(*a, **kw)


def fwd_fp8_rows(*a, **kw):
    return default().fwd_fp8_rows(*a, **kw)
