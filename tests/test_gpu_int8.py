"""INT8 scores (symmetric per-block INT8 Q and K, tcgen05.mma kind::i8) against
the oracle.

The codes and scales are integer decisions taken in fp32 on both sides, so they
must match bit for bit. The forward on the codes must match the oracle's forward
on the dequantized Q and K within the output tolerance of the bf16 path.

Against the bf16-score result the quantization itself moves the output: on these
workloads the logits reach ~25 nats, and half an INT8 step per operand adds up to
~0.02 nats per logit, about 2% of each probability. The tests hold INT8 to a
relative Frobenius distance of 5e-2 from the bf16-score oracle, and to at least 3
times less than FP8 E4M3 (whose 4 significant bits give ~11% on the same inputs)."""
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


def _int8_bytes(codes: np.ndarray) -> np.ndarray:
    return codes.astype(np.int8).view(np.uint8)


@pytest.mark.parametrize("shape", ["small", "tail"])
def test_int8_codes_and_scales_match_the_oracle_exactly(shape):
    if shape == "small":
        w = wl.WORKLOADS["small"].with_(H=4)
        q, k, _ = wl.generate(w, seed=2, device=_dev())
    else:
        q, k, _ = wl.random_qkv(2, 3, 1000, 128, seed=9, device=_dev(), scale_qk=3.0)
        q[0, 1, 64:128] = 0                                       # an all-zero block
    p8 = sa.sparse_attn_plan(q, k, 0.95, quantize="int8")
    p = sa.sparse_attn_plan(q, k, 0.95)
    torch.cuda.synchronize()
    assert sa.sparse_attn_device_error() == 0
    assert p8.qfmt == "int8"
    assert torch.equal(p8.mask, p.mask) and torch.equal(p8.work, p.work)
    for x, x8, sc in ((q, p8.q8, p8.qscale), (k, p8.k8, p8.kscale)):
        codes, scales = orc.quantize_blocks_int8(x.cpu())
        np.testing.assert_array_equal(to_np(x8), _int8_bytes(codes))
        np.testing.assert_array_equal(to_np(sc).astype(np.float64), scales)


@pytest.mark.parametrize("case,lam", [("small", None), ("small", -12.0), ("lm", None), ("tail", -6.0)])
def test_int8_score_forward_matches_the_oracle(case, lam):
    causal = case == "lm"
    if case == "small":
        w = wl.WORKLOADS["small"].with_(H=4)
        q, k, v = wl.generate(w, seed=3, device=_dev())
    elif case == "lm":
        w = wl.WORKLOADS["lm"].with_(H=2, N=2048)
        q, k, v = wl.generate(w, seed=3, device=_dev())
    else:
        q, k, v = wl.random_qkv(2, 3, 1000, 128, seed=10, device=_dev(), scale_qk=2.0)   # B = 2, ragged tail
    p = sa.sparse_attn_plan(q, k, 0.95, None, causal, quantize="int8")
    st8 = torch.zeros(4, dtype=torch.int64, device=_dev())
    st = torch.zeros(4, dtype=torch.int64, device=_dev())
    o8 = sa.sparse_attn_fwd(q, k, v, p, lam, stats=st8, qk_int8=True)
    o = sa.sparse_attn_fwd(q, k, v, p, lam, stats=st)
    torch.cuda.synchronize()
    assert sa.sparse_attn_device_error() == 0
    mask = to_np(p.mask)
    ref = orc.fwd_int8qk(q.cpu(), k.cpu(), v.cpu(), mask, lam, None, causal)
    assert_output_close(to_np(o8), ref, f"int8 scores {case} lam={lam}")
    assert int(st8[0]) == int(st[0])                         # the same kept pairs
    # the quantization's own effect, against the bf16-score oracle and against E4M3
    ref16 = orc.fwd(q.cpu(), k.cpu(), v.cpu(), mask, lam, None, causal)
    max_abs, rel = output_errors(to_np(o8), ref16)
    _, rel8 = output_errors(orc.fwd_fp8qk(q.cpu(), k.cpu(), v.cpu(), mask, lam, None, causal), ref16)
    print(f"{case} lam={lam}: int8-score output vs the bf16-score oracle max_abs={max_abs:.3e} rel_fro={rel:.3e}"
          f" (fp8 scores: rel_fro={rel8:.3e})")
    assert rel <= 5e-2 and rel * 3 <= rel8


@pytest.mark.slow
@pytest.mark.parametrize("name,tau,lam", [("hunyuan", 0.95, -12.0), ("wan", 0.95, None)])
def test_int8_scores_full_size(name, tau, lam):
    """Full size: codes and scales of a sampled head byte for byte, and 16 sampled
    query blocks (first and ragged last included) against the oracle on the
    dequantized Q and K at the output tolerance; against the bf16-score oracle
    within 5e-2 and 3 times closer than FP8 scores."""
    w = wl.WORKLOADS[name]
    q, k, v = wl.generate(w, seed=0, device=_dev())
    p = sa.sparse_attn_plan(q, k, tau, None, w.causal, quantize="int8")
    o = sa.sparse_attn_fwd(q, k, v, p, lam, qk_int8=True)
    torch.cuda.synchronize()
    assert sa.sparse_attn_device_error() == 0
    Nb = -(-w.N // 64)
    mask = to_np(p.mask)
    rng = np.random.default_rng(13)
    h = 5
    qh, kh, vh = (x[:, h:h + 1].cpu() for x in (q, k, v))
    for x, x8, sc in ((qh, p.q8, p.qscale), (kh, p.k8, p.kscale)):
        codes, scales = orc.quantize_blocks_int8(x)
        np.testing.assert_array_equal(to_np(x8[:, h:h + 1]), _int8_bytes(codes))
        np.testing.assert_array_equal(to_np(sc[:, h:h + 1]).astype(np.float64), scales)
    qbs = sorted({0, Nb - 1, *rng.choice(Nb, size=14, replace=False).tolist()})
    got = to_np(o[:, h:h + 1])
    ref = orc.fwd_int8qk(qh, kh, vh, mask[:, h:h + 1], lam, None, w.causal, qblocks=qbs)
    assert_output_close(got, ref, f"int8 {name} head {h} query blocks {qbs}")
    ref16 = orc.fwd(qh, kh, vh, mask[:, h:h + 1], lam, None, w.causal, qblocks=qbs)
    ma, rel = output_errors(got, ref16)
    _, rel8 = output_errors(orc.fwd_fp8qk(qh, kh, vh, mask[:, h:h + 1], lam, None, w.causal, qblocks=qbs), ref16)
    print(f"{name}: int8-score output vs the bf16-score oracle max_abs={ma:.3e} rel_fro={rel:.3e}"
          f" (fp8 scores: rel_fro={rel8:.3e})")
    assert rel <= 5e-2 and rel * 3 <= rel8


def test_int8_needs_an_int8_plan_and_d128():
    q, k, v = wl.random_qkv(1, 1, 256, 128, seed=1, device=_dev())
    p = sa.sparse_attn_plan(q, k, 0.9)
    with pytest.raises(ValueError):
        sa.sparse_attn_fwd(q, k, v, p, qk_int8=True)
    p8 = sa.sparse_attn_plan(q, k, 0.9, quantize="fp8")
    with pytest.raises(ValueError):
        sa.sparse_attn_fwd(q, k, v, p8, qk_int8=True)           # FP8 codes are not INT8 codes
    q64, k64, _ = wl.random_qkv(1, 1, 256, 64, seed=1, device=_dev())
    with pytest.raises(RuntimeError):
        sa.sparse_attn_plan(q64, k64, 0.9, quantize="int8")
