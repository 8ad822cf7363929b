"""The cumulative-energy (recall) P.V filter on the GPU against the oracle's
tiled-loop run of the same test (oracle.attention_recall), through the C ABI.

The GPU takes each skip decision in fp32 and records it
(sparse_attn_fwd_decisions). The oracle replays those decisions, so every
sampled output row is compared at the usual tolerance (max-abs 2e-2, relative
Frobenius 1e-2), and at every visited pair the oracle's own fp64 test must
agree with the GPU's decision unless its margin ((1 - recall) l - sk alpha - e)
/ l lies within 1e-4 of zero. The skip counts equal the recorded skips."""
import numpy as np
import pytest
import torch

from oracle import sparse_attn_oracle as orc
from tests.helpers import check_filter_replay, to_np

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import free_block_sparse_mean_b200 as sa
    from free_block_sparse_mean_b200 import workloads as wl


def _dev():
    return torch.device("cuda:0")


def _run_checked(q, k, v, plan_or_mask, recall, causal, heads=None, qblocks=None, what=""):
    """Forward with the recall filter, decisions recorded, checked head by head
    (`heads`: sampled heads, default all; `qblocks`: sampled query blocks)."""
    B, H, N, _ = q.shape
    Nb = -(-N // 64)
    stats = torch.zeros(4, dtype=torch.int64, device=_dev())
    dec = torch.zeros((B, H, Nb, Nb), dtype=torch.uint8, device=_dev())
    o = sa.sparse_attn_fwd(q, k, v, plan_or_mask, None, None, causal, recall=recall, stats=stats, decisions=dec)
    torch.cuda.synchronize()
    assert sa.sparse_attn_device_error() == 0
    mask = to_np(plan_or_mask.mask if isinstance(plan_or_mask, sa.Plan) else plan_or_mask).astype(np.uint8)
    dec_np, s = to_np(dec), to_np(stats)
    assert s[1] == int(dec_np.sum())                    # the recorded skips are the counted ones
    flips = 0
    kept = 0
    rec_min = 1.0
    for h in (range(H) if heads is None else heads):
        sl = slice(h, h + 1)
        st, f = check_filter_replay(q[:, sl].cpu(), k[:, sl].cpu(), v[:, sl].cpu(), mask[:, sl], o[:, sl],
                                    dec_np[:, sl], recall=recall, causal=causal, qblocks=qblocks,
                                    what=f"{what} head {h}")
        flips += f
        kept += st["kept_pairs"]
        rec_rows = st["recall_rows"]
        if np.isfinite(rec_rows).any():
            rec_min = min(rec_min, float(np.nanmin(rec_rows)))
    if heads is None and qblocks is None:
        assert s[0] == kept
    return int(s[1]), flips, rec_min


def _constructed(N, d, seed, aligned, a, spread):
    """Queries near a*u (u the all-ones vector), key block `aligned` near a*u
    too, every other key block noise around its own random multiple of u in
    [-spread, spread]: the blocks' shares of each row's energy spread over
    decades around the recall budget."""
    dev = _dev()
    q, k, v = wl.random_qkv(1, 2, N, d, seed=seed, device=dev)
    g = torch.Generator(device="cpu").manual_seed(seed + 1)
    Nb = -(-N // 64)
    shift = ((2 * torch.rand((1, 2, Nb, 1), generator=g) - 1) * spread).to(dev)
    u = torch.ones(d, device=dev)
    q = (q.float() * 0.5 + a * u).to(torch.bfloat16)
    kf = k.float() * 0.5 + shift.repeat_interleave(64, dim=2)[:, :, :N] * u
    al = slice(64 * aligned, 64 * aligned + 64)
    kf[:, :, al] = k.float()[:, :, al] * 0.5 + a * u
    return q, kf.to(torch.bfloat16), v


@pytest.mark.parametrize("recall,aligned,d", [(0.99, 0, 128), (0.95, 0, 128), (0.9, 7, 128), (0.97, 3, 128),
                                               (0.95, 0, 64), (0.9, 7, 64)])
def test_recall_constructed(recall, aligned, d):
    N = 1024
    a, spread = (0.6, 0.5) if d == 128 else (0.8, 0.4)
    q, k, v = _constructed(N, d, 11 + aligned, aligned, a, spread)
    Nb = N // 64
    mask = torch.ones((1, 2, Nb, Nb), dtype=torch.uint8, device=_dev())
    skipped, flips, rec_min = _run_checked(q, k, v, mask, recall, False, what=f"recall={recall}")
    assert skipped > 0
    assert rec_min >= recall - 1e-12
    print(f"recall {recall} d {d}: skipped {skipped}, decisions within the border that flipped: {flips}")


@pytest.mark.parametrize("tau,recall", [(0.95, 0.99), (0.99, 0.95)])
def test_recall_small_workload_with_plan(tau, recall):
    """The small DiT layer (H = 24, N = 4096, d = 128) with the plan's mask and tile order."""
    w = wl.WORKLOADS["small"]
    q, k, v = wl.generate(w, seed=0, device=_dev())
    p = sa.sparse_attn_plan(q, k, tau)
    _run_checked(q, k, v, p, recall, False, heads=[0, 5, 23], what=f"small tau={tau} recall={recall}")


def test_recall_causal_ragged_two_batches():
    """B = 2, causal, N = 1000 (a tail of 40 rows), d = 64, plan with tau = 0.9."""
    q, k, v = wl.random_qkv(2, 2, 1000, 64, seed=3, device=_dev())
    p = sa.sparse_attn_plan(q, k, 0.9, None, True)
    _run_checked(q, k, v, p, 0.9, True, what="causal ragged B=2")


def test_recall_one_is_the_unfiltered_forward():
    """recall = 1 skips only blocks of zero energy, whose P is zero anyway: the
    output is bit-identical to the forward without a filter."""
    w = wl.WORKLOADS["small"]
    q, k, v = wl.generate(w, seed=1, device=_dev())
    p = sa.sparse_attn_plan(q, k, 0.95)
    a = sa.sparse_attn_fwd(q, k, v, p, None)
    b = sa.sparse_attn_fwd(q, k, v, p, recall=1.0)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@pytest.mark.slow
def test_recall_full_size_sampled():
    """HunyuanVideo shape (H = 24, N = 118,800: a ragged tail), tau = 0.95, recall
    0.99, in the benchmark's launch configuration: 64 seeded query blocks plus the
    first and the ragged last of two heads, every row at the output tolerance
    under the GPU's own decisions, and the decisions against the oracle's test."""
    w = wl.WORKLOADS["hunyuan"]
    q, k, v = wl.generate(w, seed=0, device=_dev())
    p = sa.sparse_attn_plan(q, k, 0.95, None, w.causal)
    Nb = -(-w.N // 64)
    rng = np.random.default_rng(5)
    qbs = sorted({0, Nb - 1, *rng.choice(Nb, size=64, replace=False).tolist()})
    skipped, flips, _ = _run_checked(q, k, v, p, 0.99, w.causal, heads=(0, 13), qblocks=qbs,
                                     what="hunyuan recall 0.99")
    print(f"hunyuan recall 0.99: {skipped} pairs skipped; {flips} sampled decisions flipped within the border")


def test_recall_argument_errors():
    q, k, v = wl.random_qkv(1, 1, 128, 64, seed=0, device=_dev())
    mask = torch.ones((1, 1, 2, 2), dtype=torch.uint8, device=_dev())
    with pytest.raises(ValueError):
        sa.sparse_attn_fwd(q, k, v, mask, -12.0, recall=0.9)
    with pytest.raises(sa.SparseAttnError):
        sa.sparse_attn_fwd(q, k, v, mask, recall=0.0)
    with pytest.raises(sa.SparseAttnError):
        sa.sparse_attn_fwd_recall(q, k, v, mask, float("nan"))
