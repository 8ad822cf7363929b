"""Quantized scores (FP8 E4M3 Q and K, per-block scales) against the oracle.

The codes and scales are integer decisions taken in fp32 on both sides, so they
must match bit for bit; the forward on the codes must match the oracle's forward
on the dequantized Q and K within the output tolerance of the bf16 path."""
import numpy as np
import pytest
import torch

from oracle import sparse_attn_oracle as orc
from tests.helpers import assert_output_close, output_errors, to_np

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import free_block_sparse_mean_b200 as sa
    from free_block_sparse_mean_b200 import workloads as wl


def _dev():
    return torch.device("cuda:0")


def _e4m3_bytes(codes: np.ndarray) -> np.ndarray:
    return torch.tensor(codes, dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


@pytest.mark.parametrize("shape", ["small", "tail"])
def test_codes_and_scales_match_the_oracle_exactly(shape):
    if shape == "small":
        w = wl.WORKLOADS["small"].with_(H=4)
        q, k, _ = wl.generate(w, seed=2, device=_dev())
    else:
        q, k, _ = wl.random_qkv(2, 3, 1000, 128, seed=9, device=_dev(), scale_qk=3.0)
        q[0, 1, 64:128] = 0                                       # an all-zero block
    p8 = sa.sparse_attn_plan(q, k, 0.95, quantize=True)
    p = sa.sparse_attn_plan(q, k, 0.95)
    torch.cuda.synchronize()
    assert sa.sparse_attn_device_error() == 0
    assert torch.equal(p8.mask, p.mask) and torch.equal(p8.work, p.work)
    for x, x8, sc in ((q, p8.q8, p8.qscale), (k, p8.k8, p8.kscale)):
        codes, scales = orc.quantize_blocks_e4m3(x.cpu())
        np.testing.assert_array_equal(to_np(x8), _e4m3_bytes(codes))
        np.testing.assert_array_equal(to_np(sc).astype(np.float64), scales)


@pytest.mark.parametrize("case,lam", [("small", None), ("small", -12.0), ("lm", None), ("tail", -6.0)])
def test_fp8_score_forward_matches_the_oracle(case, lam):
    causal = case == "lm"
    if case == "small":
        w = wl.WORKLOADS["small"].with_(H=4)
        q, k, v = wl.generate(w, seed=3, device=_dev())
    elif case == "lm":
        w = wl.WORKLOADS["lm"].with_(H=2, N=2048)
        q, k, v = wl.generate(w, seed=3, device=_dev())
    else:
        q, k, v = wl.random_qkv(2, 3, 1000, 128, seed=10, device=_dev(), scale_qk=2.0)   # B = 2, ragged tail
    p = sa.sparse_attn_plan(q, k, 0.95, None, causal, quantize=True)
    st8 = torch.zeros(4, dtype=torch.int64, device=_dev())
    st = torch.zeros(4, dtype=torch.int64, device=_dev())
    o8 = sa.sparse_attn_fwd(q, k, v, p, lam, stats=st8, qk_fp8=True)
    o = sa.sparse_attn_fwd(q, k, v, p, lam, stats=st)
    torch.cuda.synchronize()
    assert sa.sparse_attn_device_error() == 0
    mask = to_np(p.mask)
    ref = orc.fwd_fp8qk(q.cpu(), k.cpu(), v.cpu(), mask, lam, None, causal)
    assert_output_close(to_np(o8), ref, f"fp8 scores {case} lam={lam}")
    assert int(st8[0]) == int(st[0])                         # the same kept pairs
    max_abs, rel = output_errors(to_np(o8), to_np(o).astype(np.float64))
    print(f"{case} lam={lam}: fp8-score vs bf16-score output max_abs={max_abs:.3e} rel_fro={rel:.3e}")


def test_fp8_needs_a_quantized_plan_and_d128():
    q, k, v = wl.random_qkv(1, 1, 256, 128, seed=1, device=_dev())
    p = sa.sparse_attn_plan(q, k, 0.9)
    with pytest.raises(ValueError):
        sa.sparse_attn_fwd(q, k, v, p, qk_fp8=True)
    q64, k64, _ = wl.random_qkv(1, 1, 256, 64, seed=1, device=_dev())
    with pytest.raises(RuntimeError):
        sa.sparse_attn_plan(q64, k64, 0.9, quantize=True)
