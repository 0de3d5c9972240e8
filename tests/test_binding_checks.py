"""The binding's argument checks, on the CPU: a tensor of the wrong shape,
dtype or layout, or one not on a CUDA device, is refused before any pointer
reaches the library (which reads every tensor as dense rows and cannot see
strides)."""

import pytest
import torch

from exact_io_aware_bwd_b200 import binding


def _fwd_args(B=1, Hq=4, Hkv=2, N=16, d=64, dtype=torch.bfloat16):
    q = torch.zeros((B, Hq, N, d), dtype=dtype)
    k = torch.zeros((B, Hkv, N, d), dtype=dtype)
    v = torch.zeros((B, Hkv, N, d), dtype=dtype)
    o = torch.zeros_like(q)
    lse = torch.zeros((B, Hq, N), dtype=torch.float32)
    return q, k, v, o, lse


def test_cpu_tensors_are_refused():
    q, k, v, o, lse = _fwd_args()
    with pytest.raises(ValueError, match="CUDA device"):
        binding.fa_fwd(q, k, v, o, lse, 0.1, True)


def test_strided_views_are_refused():
    q, k, v, o, lse = _fwd_args(N=16, d=64)
    qt = torch.zeros((1, 4, 64, 16), dtype=torch.bfloat16).transpose(2, 3)  # right shape, wrong layout
    with pytest.raises(ValueError, match="q must be contiguous"):
        binding.fa_fwd(qt, k, v, o, lse, 0.1, True)


@pytest.mark.parametrize("which", ["k", "v", "o"])
def test_mixed_dtypes_are_refused(which):
    args = dict(zip("q k v o lse".split(), _fwd_args()))
    args[which] = args[which].to(torch.float16)
    with pytest.raises(TypeError, match=which):
        binding.fa_fwd(args["q"], args["k"], args["v"], args["o"], args["lse"], 0.1, False)


def test_wrong_shapes_and_lse_dtype_are_refused():
    q, k, v, o, lse = _fwd_args()
    with pytest.raises(ValueError, match="v has shape"):
        binding.fa_fwd(q, k, v[:, :, :8].contiguous(), o, lse, 0.1, False)
    with pytest.raises(TypeError, match="lse"):
        binding.fa_fwd(q, k, v, o, lse.double(), 0.1, False)
    with pytest.raises(TypeError, match="q has dtype"):
        binding.fa_fwd(q.float(), k.float(), v.float(), o.float(), lse, 0.1, False)
    with pytest.raises(ValueError, match="4-D"):
        binding.fa_fwd(q[0], k[0], v[0], o[0], lse[0], 0.1, False)


def test_backward_checks_gradients_and_workspace():
    q, k, v, o, lse = _fwd_args()
    do, dq, dk, dv = torch.zeros_like(q), torch.zeros_like(q), torch.zeros_like(k), torch.zeros_like(v)
    ws = torch.zeros(1024, dtype=torch.uint8)
    with pytest.raises(ValueError, match="dk has shape"):
        binding.fa_bwd(q, k, v, o, do, lse, dq, dq, dv, 0.1, True, ws)
    with pytest.raises(ValueError, match="workspace must be contiguous"):
        binding.fa_bwd(q, k, v, o, do, lse, dq, dk, dv, 0.1, True, ws.view(32, 32).t())


def test_fp8_checks():
    B, Hq, Hkv, N, d = 1, 2, 1, 16, 128
    q8 = torch.zeros((B, Hq, N, d), dtype=torch.uint8)
    k8 = torch.zeros((B, Hkv, N, d), dtype=torch.float8_e4m3fn)
    v8 = torch.zeros((B, Hkv, N, d), dtype=torch.uint8)
    o = torch.zeros((B, Hq, N, d), dtype=torch.bfloat16)
    lse = torch.zeros((B, Hq, N), dtype=torch.float32)
    with pytest.raises(ValueError, match="CUDA device"):
        binding.fa_fwd_fp8(q8, k8, v8, o, lse, 0.1, (1.0, 1.0, 1.0), True)
    with pytest.raises(TypeError, match="q8 has dtype"):
        binding.fa_fwd_fp8(q8.to(torch.bfloat16), k8, v8, o, lse, 0.1, (1.0, 1.0, 1.0), True)
    with pytest.raises(TypeError, match="o must be"):
        binding.fa_fwd_fp8(q8, k8, v8, o.float(), lse, 0.1, (1.0, 1.0, 1.0), True)
