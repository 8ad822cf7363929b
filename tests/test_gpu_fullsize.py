"""Parity at the full workload sizes, in the launch configuration the benchmark
times (plan with the tile order, forward over the plan's pairs).

Masks: every head (every 4th for the extra centroid weights) against the
oracle's plan (exact outside the 1e-4 band).
Outputs: the oracle run with the GPU's own mask on 64 seeded query blocks plus
the first and the last (the ragged tail when N % 64 != 0) of the sampled heads;
each query block's output is independent given the mask, so the sampled rows
are exact comparisons. With lambda the oracle replays the GPU's recorded skip
decisions, and each decision is checked against the oracle's own test."""
import numpy as np
import pytest
import torch

from oracle import sparse_attn_oracle as orc
from tests.helpers import (assert_output_close, check_filter_replay, check_plan_consistency, compare_masks,
                           output_errors, to_np)

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

if torch.cuda.is_available():
    import free_block_sparse_mean_b200 as sa
    from free_block_sparse_mean_b200 import workloads as wl

SAMPLED_QBLOCKS = 64

CASES = [
    # workload, tau, lambda, centroid weight, heads whose outputs are sampled, mask-head stride
    ("wan", 0.95, None, None, (0, 23), 1),
    ("hunyuan", 0.90, -12.0, 0.5, (9,), 4),
    ("hunyuan", 0.90, -12.0, 1.5, (2,), 4),
    ("hunyuan", 0.90, -12.0, 3.0, (5,), 4),
    ("hunyuan", 0.95, -12.0, 0.5, (7,), 4),
    ("hunyuan", 0.95, -12.0, 1.5, (0, 17), 1),
    ("hunyuan", 0.95, -12.0, 3.0, (21,), 4),
    ("lm", 0.95, None, None, (0, 31), 1),
]


def sampled_qblocks(Nb, seed):
    rng = np.random.default_rng(seed)
    return sorted({0, Nb - 1, *rng.choice(Nb, size=min(Nb, SAMPLED_QBLOCKS), replace=False).tolist()})


@pytest.mark.parametrize("name,tau,lam,cw,out_heads,stride", CASES)
def test_full_size_masks_and_sampled_outputs(name, tau, lam, cw, out_heads, stride):
    dev = torch.device("cuda:0")
    w = wl.WORKLOADS[name]
    q, k, v = wl.generate(w, seed=0, device=dev, centroid_weight=cw)
    Nb = -(-w.N // 64)
    plan = sa.sparse_attn_plan(q, k, tau, None, w.causal, with_idx=True)
    dec = torch.zeros((w.B, w.H, Nb, Nb), dtype=torch.uint8, device=dev)
    out = sa.sparse_attn_fwd(q, k, v, plan, lam, decisions=dec)
    torch.cuda.synchronize()
    assert sa.sparse_attn_device_error() == 0
    mask = to_np(plan.mask)
    check_plan_consistency(mask[0, :2], to_np(plan.count)[0, :2], to_np(plan.idx)[0, :2])
    del plan
    rows_diff = excused = 0
    heads = range(0, w.H, stride)
    for h in heads:
        qh, kh = q[:, h:h + 1].cpu(), k[:, h:h + 1].cpu()
        op = orc.plan(qh, kh, tau, None, w.causal)
        r, e = compare_masks(mask[:, h:h + 1], op, tau)
        rows_diff += r
        excused += e
    print(f"{name} tau={tau} cw={cw}: rows differing {rows_diff} of {len(heads) * Nb}, excused blocks {excused}, "
          f"density {mask.mean():.3f}")
    assert rows_diff <= max(2, (len(heads) * Nb) // 500)
    dec_np = to_np(dec) if lam is not None else None
    for h in out_heads:
        qbs = sampled_qblocks(Nb, 7 + h)
        qh, kh, vh = (x[:, h:h + 1].cpu() for x in (q, k, v))
        got = to_np(out[:, h:h + 1])
        if lam is None:
            ref = orc.fwd(qh, kh, vh, mask[:, h:h + 1], None, None, w.causal, qblocks=qbs)
            assert_output_close(got, ref, f"{name} head {h}, {len(qbs)} query blocks")
        else:
            _, flips = check_filter_replay(qh, kh, vh, mask[:, h:h + 1], got, dec_np[:, h:h + 1], lam=lam,
                                           causal=w.causal, qblocks=qbs,
                                           what=f"{name} cw={cw} head {h}, {len(qbs)} query blocks")
            print(f"  head {h}: {flips} lambda decisions flipped within the border")
        dense = orc.attention_masked(qh, kh, vh, np.ones((1, 1, Nb, Nb), np.uint8), None, w.causal,
                                     qblocks=qbs[:8])
        ma, rel = output_errors(got, dense)
        print(f"  head {h}: sparse-vs-dense on 8 query blocks max_abs={ma:.3e} rel_fro={rel:.3e}")


def test_full_mask_natural_pairs_repeated():
    """Full mask over every key block, tiles in natural order (no plan), on the
    peaked HunyuanVideo data (centroid weight 3): long union lists with S(k+1)
    already resident while P(k) is published, repeated so a barrier-phase race
    would show as a device-side timeout. Sampled rows against the oracle."""
    dev = torch.device("cuda:0")
    w = wl.WORKLOADS["hunyuan"]
    q, k, v = wl.generate(w, seed=0, device=dev, centroid_weight=3.0)
    Nb = -(-w.N // 64)
    full = torch.ones((w.B, w.H, Nb, Nb), dtype=torch.uint8, device=dev)
    out = torch.empty_like(q)
    for _ in range(3):
        sa.sparse_attn_fwd(q, k, v, full, None, out=out, causal=w.causal)
        torch.cuda.synchronize()
        assert sa.sparse_attn_device_error() == 0
    h = 11
    qbs = [0, 777, Nb - 1]
    qh, kh, vh = (x[:, h:h + 1].cpu() for x in (q, k, v))
    ones = np.ones((1, 1, Nb, Nb), dtype=np.uint8)
    ref = orc.fwd(qh, kh, vh, ones, None, None, w.causal, qblocks=qbs)
    assert_output_close(to_np(out[:, h:h + 1]), ref, f"full mask head {h} query blocks {qbs}")


@pytest.mark.parametrize("name,tau,lam,out_heads", [("hunyuan", 0.95, -12.0, (3,)), ("wan", 0.95, None, (7,))])
def test_full_size_fp8_scores(name, tau, lam, out_heads):
    """The quantized-score variant at full size: the codes and scales of sampled
    heads byte for byte against the oracle's quantizer, and sampled query blocks of
    the forward on the codes against the oracle on the dequantized Q and K."""
    dev = torch.device("cuda:0")
    w = wl.WORKLOADS[name]
    q, k, v = wl.generate(w, seed=0, device=dev)
    plan = sa.sparse_attn_plan(q, k, tau, None, w.causal, quantize=True)
    out = sa.sparse_attn_fwd(q, k, v, plan, lam, qk_fp8=True)
    torch.cuda.synchronize()
    assert sa.sparse_attn_device_error() == 0
    Nb = -(-w.N // 64)
    mask = to_np(plan.mask)
    rng = np.random.default_rng(11)
    for h in out_heads:
        qh, kh, vh = (x[:, h:h + 1].cpu() for x in (q, k, v))
        for x, x8, sc in ((qh, plan.q8, plan.qscale), (kh, plan.k8, plan.kscale)):
            codes, scales = orc.quantize_blocks_e4m3(x)
            want = torch.tensor(codes, dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
            np.testing.assert_array_equal(to_np(x8[:, h:h + 1]), want)
            np.testing.assert_array_equal(to_np(sc[:, h:h + 1]).astype(np.float64), scales)
        qbs = sorted({0, Nb - 1, *rng.choice(Nb, size=4, replace=False).tolist()})
        ref = orc.fwd_fp8qk(qh, kh, vh, mask[:, h:h + 1], lam, None, w.causal, qblocks=qbs)
        assert_output_close(to_np(out[:, h:h + 1]), ref, f"fp8 {name} head {h} query blocks {qbs}")
