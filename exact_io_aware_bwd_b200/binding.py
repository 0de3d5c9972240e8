"""ctypes binding of libfa_b200.so: the C ABI of include/fa.h, one Python
function per entry point with the same name, plus two conveniences that
allocate outputs with PyTorch.  Argument marshalling only: every step of the
computation runs in the library's CUDA kernels.  There is no fallback: if the
library cannot be loaded, every call raises.
"""

from __future__ import annotations

import ctypes
import math
import os
import threading

import torch

from .build import LIB_PATH

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_MISALIGNED, FA_ERR_CUDA, FA_ERR_TIMEOUT = range(6)
FA_BF16, FA_FP16 = 0, 1

_DTYPES = {torch.bfloat16: FA_BF16, torch.float16: FA_FP16}

_lock = threading.Lock()
_lib = None


class FaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {fa_status_string(status)} (status {status})")


def library_path() -> str:
    return os.environ.get("FA_B200_LIB", LIB_PATH)


def load():
    """Load libfa_b200.so (built in-tree by build.build()); raise if absent."""
    global _lib
    with _lock:
        if _lib is None:
            path = library_path()
            if not os.path.exists(path):
                raise RuntimeError(
                    f"{path} is missing: build it with exact_io_aware_bwd_b200.build.build() "
                    "(there is no fallback implementation)")
            lib = ctypes.CDLL(path)
            vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
            lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp]
            lib.fa_fwd.restype = i
            lib.fa_bwd_workspace_bytes.argtypes = [i, i, i, i, i]
            lib.fa_bwd_workspace_bytes.restype = ctypes.c_size_t
            lib.fa_bwd.argtypes = ([vp] * 9 + [i, i, i, i, i, f, i, i, vp, ctypes.c_size_t, vp])
            lib.fa_bwd.restype = i
            lib.fa_fwd_window.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp]
            lib.fa_fwd_window.restype = i
            lib.fa_bwd_window.argtypes = ([vp] * 9 + [i, i, i, i, i, f, i, i, vp, ctypes.c_size_t, vp])
            lib.fa_bwd_window.restype = i
            u64 = ctypes.c_uint64
            lib.fa_fwd_dropout.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, f, u64, i, vp]
            lib.fa_fwd_dropout.restype = i
            lib.fa_bwd_dropout.argtypes = ([vp] * 9 + [i, i, i, i, i, f, i, f, u64, i, vp,
                                                       ctypes.c_size_t, vp])
            lib.fa_bwd_dropout.restype = i
            lib.fa_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, f, f, f, i, i, vp]
            lib.fa_fwd_fp8.restype = i
            lib.fa_fwd_blockmask.argtypes = [vp] * 5 + [i] * 5 + [f, i, vp, i, i, vp]
            lib.fa_fwd_blockmask.restype = i
            lib.fa_bwd_blockmask_workspace_bytes.argtypes = [i, i, i, i, i]
            lib.fa_bwd_blockmask_workspace_bytes.restype = ctypes.c_size_t
            lib.fa_bwd_blockmask.argtypes = ([vp] * 9 + [i] * 5 + [f, i, vp, i, i, vp, ctypes.c_size_t, vp])
            lib.fa_bwd_blockmask.restype = i
            lib.fa_decode_workspace_bytes.argtypes = [i, i, i, i, i, i]
            lib.fa_decode_workspace_bytes.restype = ctypes.c_size_t
            lib.fa_decode_paged.argtypes = ([vp] * 7 + [i] * 8 + [f, i, vp, ctypes.c_size_t, vp])
            lib.fa_decode_paged.restype = i
            lib.fa_get_device_status.argtypes = [vp]
            lib.fa_get_device_status.restype = i
            lib.fa_peek_device_status_word.argtypes = [vp]
            lib.fa_peek_device_status_word.restype = ctypes.c_uint32
            lib.fa_selftest_wait_timeout.argtypes = [ctypes.c_uint64, vp]
            lib.fa_selftest_wait_timeout.restype = i
            lib.fa_set_profile_events.argtypes = [i, vp, vp]
            lib.fa_set_profile_events.restype = i
            lib.fa_set_bwd_max_blocks.argtypes = [i]
            lib.fa_set_bwd_max_blocks.restype = i
            lib.fa_status_string.argtypes = [i]
            lib.fa_status_string.restype = ctypes.c_char_p
            _lib = lib
    return _lib


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return ctypes.c_void_p(t)
    return ctypes.c_void_p(t.data_ptr())


def _check(status: int, where: str):
    if status != FA_OK:
        raise FaError(status, where)


def _dims(q, k):
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError(f"q and k must be 4-D [B, H, N, d], got {tuple(q.shape)} and {tuple(k.shape)}")
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    return B, Hq, Hkv, N, d


_E4M3 = (torch.uint8, torch.float8_e4m3fn)


def _expect(where, *spec):
    """Checks (name, tensor, shape, dtypes) entries before any pointer reaches
    the library: the shape (None: any), the dtype (None: any), a dense
    row-major layout, and one CUDA device for all.  The library reads every
    tensor as dense rows, so a strided view would be read wrongly rather than
    rejected there.  None and raw integer addresses pass through unchecked."""
    spec = [(name, t, shape, dtypes) for name, t, shape, dtypes in spec
            if t is not None and not isinstance(t, int)]
    for name, t, shape, dtypes in spec:
        if shape is not None and tuple(t.shape) != tuple(shape):
            raise ValueError(f"{where}: {name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
        if dtypes is not None and t.dtype not in dtypes:
            raise TypeError(f"{where}: {name} has dtype {t.dtype}, expected one of {list(dtypes)}")
        if not t.is_contiguous():
            raise ValueError(f"{where}: {name} must be contiguous")
    dev = None
    for name, t, _, _ in spec:
        if not t.is_cuda:
            raise ValueError(f"{where}: {name} must be on a CUDA device")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"{where}: all tensors must be on one device ({name} is on {t.device})")


def _expect_attention(where, q, k, v, o, lse, dout=None, dq=None, dk=None, dv=None, workspace=None):
    """_expect for the attention entry points; returns (B, Hq, Hkv, N, d)."""
    B, Hq, Hkv, N, d = _dims(q, k)
    if q.dtype not in _DTYPES:
        raise TypeError(f"{where}: q has dtype {q.dtype}, expected bfloat16 or float16")
    same = (q.dtype,)
    qs, ks = (B, Hq, N, d), (B, Hkv, N, d)
    _expect(where, ("q", q, qs, same), ("k", k, ks, same), ("v", v, ks, same), ("o", o, qs, same),
            ("lse", lse, (B, Hq, N), (torch.float32,)), ("dout", dout, qs, same),
            ("dq", dq, qs, same), ("dk", dk, ks, same), ("dv", dv, ks, same),
            ("workspace", workspace, None, None))
    return B, Hq, Hkv, N, d


def fa_status_string(status: int) -> str:
    return load().fa_status_string(int(status)).decode()


def fa_fwd(q, k, v, o, lse, scale: float, causal: bool, stream=None) -> None:
    """O and lse (natural log) of exact attention into the given tensors.
    q [B,Hq,N,d], k/v [B,Hkv,N,d] (bf16 or fp16, contiguous, on the GPU)."""
    B, Hq, Hkv, N, d = _expect_attention("fa_fwd", q, k, v, o, lse)
    st = load().fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, N, d,
                       float(scale), int(bool(causal)), _DTYPES[q.dtype], _stream(stream))
    _check(st, "fa_fwd")


def fa_fwd_window(q, k, v, o, lse, scale: float, window: int, stream=None) -> None:
    """Causal sliding-window forward: query i sees keys i-window+1 .. i."""
    B, Hq, Hkv, N, d = _expect_attention("fa_fwd_window", q, k, v, o, lse)
    st = load().fa_fwd_window(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, N, d,
                              float(scale), int(window), _DTYPES[q.dtype], _stream(stream))
    _check(st, "fa_fwd_window")


def fa_bwd_window(q, k, v, o, dout, lse, dq, dk, dv, scale: float, window: int, workspace,
                  stream=None) -> None:
    """Backward of fa_fwd_window with the same window."""
    B, Hq, Hkv, N, d = _expect_attention("fa_bwd_window", q, k, v, o, lse, dout, dq, dk, dv, workspace)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = load().fa_bwd_window(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq),
                              _ptr(dk), _ptr(dv), B, Hq, Hkv, N, d, float(scale), int(window),
                              _DTYPES[q.dtype], _ptr(workspace), ws_bytes, _stream(stream))
    _check(st, "fa_bwd_window")


def fa_fwd_dropout(q, k, v, o, lse, scale: float, causal: bool, p_drop: float, seed: int,
                   stream=None) -> None:
    """Forward with dropout on the probabilities (8-bit threshold round(256 p))."""
    B, Hq, Hkv, N, d = _expect_attention("fa_fwd_dropout", q, k, v, o, lse)
    st = load().fa_fwd_dropout(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, N, d,
                               float(scale), int(bool(causal)), float(p_drop),
                               int(seed) & 0xFFFFFFFFFFFFFFFF, _DTYPES[q.dtype], _stream(stream))
    _check(st, "fa_fwd_dropout")


def fa_fwd_fp8(q8, k8, v8, o, lse, scale: float, descale, causal: bool, stream=None) -> None:
    """FP8 forward: q8 [B,Hq,N,128], k8/v8 [B,Hkv,N,128] E4M3 codes (uint8 or
    float8_e4m3fn tensors on the GPU), descale = (delta_q, delta_k, delta_v);
    O (bf16 or fp16, its dtype picks the output type) and lse fp32."""
    B, Hq, Hkv, N, d = _dims(q8, k8)
    if o is None or isinstance(o, int) or o.dtype not in _DTYPES:
        raise TypeError("fa_fwd_fp8: o must be a bfloat16 or float16 tensor (its dtype picks the output type)")
    _expect("fa_fwd_fp8", ("q8", q8, (B, Hq, N, d), _E4M3), ("k8", k8, (B, Hkv, N, d), _E4M3),
            ("v8", v8, (B, Hkv, N, d), _E4M3), ("o", o, (B, Hq, N, d), None),
            ("lse", lse, (B, Hq, N), (torch.float32,)))
    dq, dk, dv = (float(x) for x in descale)
    st = load().fa_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(o), _ptr(lse), B, Hq, Hkv, N, d,
                           float(scale), dq, dk, dv, int(bool(causal)), _DTYPES[o.dtype],
                           _stream(stream))
    _check(st, "fa_fwd_fp8")


def attention_fwd_fp8(q8, k8, v8, descale, scale: float | None = None, causal: bool = False,
                      out_dtype=torch.bfloat16, stream=None):
    """Allocates O (out_dtype) and lse and runs fa_fwd_fp8; returns (O, lse)."""
    B, Hq, Hkv, N, d = _dims(q8, k8)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o = torch.empty((B, Hq, N, d), device=q8.device, dtype=out_dtype)
    lse = torch.empty((B, Hq, N), device=q8.device, dtype=torch.float32)
    fa_fwd_fp8(q8, k8, v8, o, lse, scale, descale, causal, stream)
    return o, lse


def fa_bwd_dropout(q, k, v, o, dout, lse, dq, dk, dv, scale: float, causal: bool, p_drop: float,
                   seed: int, workspace, stream=None) -> None:
    """Backward of fa_fwd_dropout with the same p_drop and seed."""
    B, Hq, Hkv, N, d = _expect_attention("fa_bwd_dropout", q, k, v, o, lse, dout, dq, dk, dv, workspace)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = load().fa_bwd_dropout(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq),
                               _ptr(dk), _ptr(dv), B, Hq, Hkv, N, d, float(scale),
                               int(bool(causal)), float(p_drop), int(seed) & 0xFFFFFFFFFFFFFFFF,
                               _DTYPES[q.dtype], _ptr(workspace), ws_bytes, _stream(stream))
    _check(st, "fa_bwd_dropout")


def _block_mask(where, block_mask, Hq, N, device):
    """(tensor, mask_per_head) of a block mask over 128 x 128 blocks: a bool
    or uint8 CUDA tensor [nb, nb] (every head) or [Hq, nb, nb], nb = ceil(N/128)."""
    nb = -(-N // 128)
    if block_mask is None or isinstance(block_mask, int):
        raise ValueError(f"{where}: a block mask tensor is required")
    if block_mask.dtype not in (torch.uint8, torch.bool):
        raise TypeError(f"{where}: block_mask has dtype {block_mask.dtype}, expected uint8 or bool")
    if tuple(block_mask.shape) == (nb, nb):
        per_head = 0
    elif tuple(block_mask.shape) == (Hq, nb, nb):
        per_head = 1
    else:
        raise ValueError(f"{where}: block_mask has shape {tuple(block_mask.shape)}, expected "
                         f"({nb}, {nb}) or ({Hq}, {nb}, {nb})")
    if not block_mask.is_cuda or block_mask.device != device:
        raise ValueError(f"{where}: block_mask must be on {device}")
    if not block_mask.is_contiguous():
        raise ValueError(f"{where}: block_mask must be contiguous")
    return block_mask.view(torch.uint8) if block_mask.dtype == torch.bool else block_mask, per_head


def fa_fwd_blockmask(q, k, v, o, lse, scale: float, causal: bool, block_mask, stream=None) -> None:
    """Forward under a block mask over 128-row x 128-key blocks (see
    _block_mask for its layout); combined with the causal mask when causal."""
    B, Hq, Hkv, N, d = _expect_attention("fa_fwd_blockmask", q, k, v, o, lse)
    m, per_head = _block_mask("fa_fwd_blockmask", block_mask, Hq, N, q.device)
    st = load().fa_fwd_blockmask(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, N, d,
                                 float(scale), int(bool(causal)), _ptr(m), per_head, _DTYPES[q.dtype],
                                 _stream(stream))
    _check(st, "fa_fwd_blockmask")


def fa_bwd_blockmask_workspace_bytes(B: int, Hq: int, Hkv: int, N: int, d: int) -> int:
    return int(load().fa_bwd_blockmask_workspace_bytes(B, Hq, Hkv, N, d))


def fa_bwd_blockmask(q, k, v, o, dout, lse, dq, dk, dv, scale: float, causal: bool, block_mask,
                     workspace, stream=None) -> None:
    """Backward of fa_fwd_blockmask with the same mask; workspace of at least
    fa_bwd_blockmask_workspace_bytes(...) bytes."""
    B, Hq, Hkv, N, d = _expect_attention("fa_bwd_blockmask", q, k, v, o, lse, dout, dq, dk, dv,
                                         workspace)
    m, per_head = _block_mask("fa_bwd_blockmask", block_mask, Hq, N, q.device)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = load().fa_bwd_blockmask(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq),
                                 _ptr(dk), _ptr(dv), B, Hq, Hkv, N, d, float(scale), int(bool(causal)),
                                 _ptr(m), per_head, _DTYPES[q.dtype], _ptr(workspace), ws_bytes,
                                 _stream(stream))
    _check(st, "fa_bwd_blockmask")


def fa_bwd_workspace_bytes(B: int, Hq: int, Hkv: int, N: int, d: int) -> int:
    return int(load().fa_bwd_workspace_bytes(B, Hq, Hkv, N, d))


def fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, scale: float, causal: bool, workspace,
           stream=None) -> None:
    """dQ, dK, dV into the given tensors; workspace: a uint8 GPU tensor of at
    least fa_bwd_workspace_bytes(...) bytes."""
    B, Hq, Hkv, N, d = _expect_attention("fa_bwd", q, k, v, o, lse, dout, dq, dk, dv, workspace)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = load().fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq),
                       _ptr(dk), _ptr(dv), B, Hq, Hkv, N, d, float(scale), int(bool(causal)),
                       _DTYPES[q.dtype], _ptr(workspace), ws_bytes, _stream(stream))
    _check(st, "fa_bwd")


def fa_get_device_status(stream=None) -> int:
    return int(load().fa_get_device_status(_stream(stream)))


def fa_peek_device_status_word(stream=None) -> int:
    return int(load().fa_peek_device_status_word(_stream(stream)))


def fa_selftest_wait_timeout(limit_ns: int, stream=None) -> int:
    return int(load().fa_selftest_wait_timeout(int(limit_ns), _stream(stream)))


KERNEL_FWD, KERNEL_BWD_MAIN = 1, 3


def fa_set_profile_events(kernel_id: int, start=None, stop=None) -> None:
    """Bracket every launch of a kernel with two CUDA events (torch.cuda.Event
    objects that have been recorded once, or raw handles); None clears."""
    h = lambda e: None if e is None else ctypes.c_void_p(e.cuda_event if hasattr(e, "cuda_event") else int(e))
    _check(load().fa_set_profile_events(int(kernel_id), h(start), h(stop)), "fa_set_profile_events")


def fa_set_bwd_max_blocks(max_blocks: int) -> None:
    """Cap the persistent blocks of the backward main pass (0: one per SM)."""
    _check(load().fa_set_bwd_max_blocks(int(max_blocks)), "fa_set_bwd_max_blocks")


def fa_decode_workspace_bytes(B: int, Hq: int, Hkv: int, Nq: int, d: int, max_pages: int) -> int:
    return int(load().fa_decode_workspace_bytes(B, Hq, Hkv, Nq, d, max_pages))


def fa_decode_paged(q, k_cache, v_cache, block_table, seq_lens, o, lse, scale: float, workspace,
                    stream=None) -> None:
    """Decode over a paged cache: q [B,Hq,Nq,d]; caches [pages,Hkv,P,d];
    block_table [B,max_pages] and seq_lens [B] int32 on the GPU."""
    B, Hq, Nq, d = q.shape
    num_pages, Hkv, P, dk = k_cache.shape
    if dk != d or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError(f"incompatible shapes q{tuple(q.shape)} k_cache{tuple(k_cache.shape)}")
    if block_table.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise ValueError("block_table and seq_lens must be int32")
    if q.dtype not in _DTYPES:
        raise TypeError(f"fa_decode_paged: q has dtype {q.dtype}, expected bfloat16 or float16")
    same = (q.dtype,)
    _expect("fa_decode_paged", ("q", q, None, same), ("k_cache", k_cache, None, same),
            ("v_cache", v_cache, None, same), ("block_table", block_table, (B, block_table.shape[-1]), None),
            ("seq_lens", seq_lens, (B,), None), ("o", o, (B, Hq, Nq, d), same),
            ("lse", lse, (B, Hq, Nq), (torch.float32,)), ("workspace", workspace, None, None))
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = load().fa_decode_paged(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                _ptr(seq_lens), _ptr(o), _ptr(lse), B, Hq, Hkv, Nq, d, P,
                                block_table.shape[1], num_pages, float(scale), _DTYPES[q.dtype],
                                _ptr(workspace), ws_bytes, _stream(stream))
    _check(st, "fa_decode_paged")


# ------------------------------------------------------------ conveniences

def attention_decode_paged(q, k_cache, v_cache, block_table, seq_lens, scale: float | None = None,
                           stream=None):
    """Allocates O, lse and the workspace and runs fa_decode_paged."""
    B, Hq, Nq, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, Nq), device=q.device, dtype=torch.float32)
    ws = torch.empty(max(fa_decode_workspace_bytes(B, Hq, k_cache.shape[1], Nq, d,
                                                   block_table.shape[1]), 16),
                     device=q.device, dtype=torch.uint8)
    fa_decode_paged(q, k_cache, v_cache, block_table, seq_lens, o, lse, scale, ws, stream)
    return o, lse



def attention_fwd(q, k, v, scale: float | None = None, causal: bool = False, stream=None,
                  window: int = 0, dropout=None, block_mask=None):
    """Allocates O and lse with PyTorch and runs fa_fwd (fa_fwd_window when
    window > 0, which implies causal; fa_fwd_dropout when dropout = (p_drop,
    seed); fa_fwd_blockmask when block_mask is given); returns (O, lse)."""
    if sum((bool(window), bool(dropout), block_mask is not None)) > 1:
        raise ValueError("a sliding window, dropout and a block mask are not combined")
    B, Hq, Hkv, N, d = _dims(q, k)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, N), device=q.device, dtype=torch.float32)
    if block_mask is not None:
        fa_fwd_blockmask(q, k, v, o, lse, scale, causal, block_mask, stream)
    elif window:
        fa_fwd_window(q, k, v, o, lse, scale, window, stream)
    elif dropout:
        fa_fwd_dropout(q, k, v, o, lse, scale, causal, dropout[0], dropout[1], stream)
    else:
        fa_fwd(q, k, v, o, lse, scale, causal, stream)
    return o, lse


def attention_bwd(q, k, v, o, dout, lse, scale: float | None = None, causal: bool = False,
                  workspace=None, stream=None, window: int = 0, dropout=None, block_mask=None):
    """Allocates dQ, dK, dV (and the workspace if not given) and runs fa_bwd
    (fa_bwd_window when window > 0, fa_bwd_dropout with dropout,
    fa_bwd_blockmask with a block mask)."""
    B, Hq, Hkv, N, d = _dims(q, k)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    if workspace is None:
        nbytes = (fa_bwd_blockmask_workspace_bytes(B, Hq, Hkv, N, d) if block_mask is not None
                  else fa_bwd_workspace_bytes(B, Hq, Hkv, N, d))
        workspace = torch.empty(max(nbytes, 16), device=q.device, dtype=torch.uint8)
    if block_mask is not None:
        fa_bwd_blockmask(q, k, v, o, dout, lse, dq, dk, dv, scale, causal, block_mask, workspace, stream)
    elif window:
        fa_bwd_window(q, k, v, o, dout, lse, dq, dk, dv, scale, window, workspace, stream)
    elif dropout:
        fa_bwd_dropout(q, k, v, o, dout, lse, dq, dk, dv, scale, causal, dropout[0], dropout[1],
                       workspace, stream)
    else:
        fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, scale, causal, workspace, stream)
    return dq, dk, dv


def fa_bwd_noalloc(q, k, v, o, dout, lse, dq, dk, dv, scale: float, causal: bool,
                   stream=None) -> None:
    """fa_bwd without a workspace: for callers that cannot allocate device
    memory.  Uses the library's fixed scratch array (FA_BWD_NOALLOC_SCRATCH_BYTES
    per device); raises FaError(FA_ERR_UNSUPPORTED) for problems that need more.
    Calls on one device share that array, so order them on one stream."""
    lib = load()
    fn = lib.fa_bwd_noalloc
    if fn.argtypes is None:
        vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        fn.argtypes = [vp] * 9 + [i, i, i, i, i, f, i, i, vp]
        fn.restype = i
    B, Hq, Hkv, N, d = _expect_attention("fa_bwd_noalloc", q, k, v, o, lse, dout, dq, dk, dv)
    st = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
            _ptr(dv), B, Hq, Hkv, N, d, float(scale), int(bool(causal)), _DTYPES[q.dtype],
            _stream(stream))
    _check(st, "fa_bwd_noalloc")
