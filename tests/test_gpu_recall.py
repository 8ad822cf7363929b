"""The cumulative-energy (recall) P.V filter on the GPU against the oracle's
tiled-loop run of the same test (oracle.attention_recall), through the C ABI.

The GPU takes each skip decision in fp32; it may differ from the oracle's fp64
decision only where the oracle's margin ((1 - recall) l - sk alpha - e) / l is
within rounding of zero (|margin| < 1e-4 here, far above fp32 rounding of the
sums). A flip changes sk, so the later decisions of that query block may differ
too: such a query block is excused from the strict comparison, and both outputs
then lie within (1 - recall) max|V| of the unfiltered one, so they differ by at
most twice that. Every other query block must match to the usual tolerance
(max-abs 2e-2, relative Frobenius 1e-2), and the skip counts may differ by at
most the number of decisions from the first borderline one on in the excused
query blocks."""
import numpy as np
import pytest
import torch

from oracle import sparse_attn_oracle as orc
from tests.helpers import assert_output_close, to_np

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import free_block_sparse_mean_b200 as sa
    from free_block_sparse_mean_b200 import workloads as wl

BORDER = 1e-4     # |margin| below this: the fp32 and fp64 decisions may differ


def _dev():
    return torch.device("cuda:0")


def _check_against_oracle(q, k, v, mask_np, recall, causal, o_gpu, stats_gpu, qblocks=None,
                          max_excused_frac=0.25):
    ref, st = orc.attention_recall(q.cpu(), k.cpu(), v.cpu(), mask_np, recall, None, causal,
                                   qblocks=qblocks, return_stats=True)
    got = to_np(o_gpu)
    B, H, N, _ = q.shape
    excused, cascade = set(), 0
    for b, h, i, j, skipped, margin in st["decisions"]:
        if (b, h, i) in excused or abs(margin) < BORDER:
            excused.add((b, h, i))
            cascade += 1
    vmax = float(np.abs(to_np(v)).max())
    strict = np.isfinite(ref)
    for b, h, i in excused:
        rows = slice(i * 64, min(N, i * 64 + 64))
        diff = np.abs(got[b, h, rows] - ref[b, h, rows]).max()
        assert diff <= 2e-2 + 2 * (1 - recall) * vmax, (b, h, i, diff)
        strict[b, h, rows] = False
    assert_output_close(got, np.where(strict, ref, np.nan), f"recall={recall}")
    n_q = len(list(qblocks)) * B * H if qblocks is not None else B * H * (-(-N // 64))
    assert len(excused) <= max(2, int(n_q * max_excused_frac)), f"{len(excused)} of {n_q} query blocks excused"
    if stats_gpu is not None:
        s = to_np(stats_gpu)
        assert s[0] == st["kept_pairs"]
        assert abs(int(s[1]) - st["pv_skipped"]) <= cascade
        return int(s[1]), st
    return None, st


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
    stats = torch.zeros(4, dtype=torch.int64, device=_dev())
    o = sa.sparse_attn_fwd(q, k, v, mask, recall=recall, stats=stats)
    torch.cuda.synchronize()
    assert sa.sparse_attn_device_error() == 0
    skipped, st = _check_against_oracle(q, k, v, to_np(mask).astype(np.uint8), recall, False, o, stats)
    assert skipped > 0
    assert np.nanmin(st["recall_rows"]) >= recall - 1e-12


@pytest.mark.parametrize("tau,recall", [(0.95, 0.99), (0.99, 0.95)])
def test_recall_small_workload_with_plan(tau, recall):
    """The small DiT layer (H = 24, N = 4096, d = 128) with the plan's mask and tile order."""
    w = wl.WORKLOADS["small"]
    q, k, v = wl.generate(w, seed=0, device=_dev())
    p = sa.sparse_attn_plan(q, k, tau)
    stats = torch.zeros(4, dtype=torch.int64, device=_dev())
    o = sa.sparse_attn_fwd(q, k, v, p, recall=recall, stats=stats)
    torch.cuda.synchronize()
    assert sa.sparse_attn_device_error() == 0
    heads = [0, 5, 23]
    mask = to_np(p.mask).astype(np.uint8)
    for h in heads:
        sl = slice(h, h + 1)
        _check_against_oracle(q[:, sl], k[:, sl], v[:, sl], mask[:, sl], recall, False, o[:, sl], None)


def test_recall_causal_ragged_two_batches():
    """B = 2, causal, N = 1000 (a tail of 40 rows), d = 64, plan with tau = 0.9."""
    q, k, v = wl.random_qkv(2, 2, 1000, 64, seed=3, device=_dev())
    p = sa.sparse_attn_plan(q, k, 0.9, None, True)
    stats = torch.zeros(4, dtype=torch.int64, device=_dev())
    o = sa.sparse_attn_fwd(q, k, v, p, recall=0.9, stats=stats)
    torch.cuda.synchronize()
    assert sa.sparse_attn_device_error() == 0
    _check_against_oracle(q, k, v, to_np(p.mask).astype(np.uint8), 0.9, True, o, stats)


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
    0.99, in the benchmark's launch configuration; sampled query blocks of two
    heads against the oracle. Rows this long fill their budget over hundreds of
    small blocks, so most query blocks meet a decision within 1e-4 of the
    threshold somewhere along the row: those are held to the 2 (1 - recall) max|V|
    bound, the rest to the usual tolerance."""
    w = wl.WORKLOADS["hunyuan"]
    q, k, v = wl.generate(w, seed=0, device=_dev())
    p = sa.sparse_attn_plan(q, k, 0.95, None, w.causal)
    o = sa.sparse_attn_fwd(q, k, v, p, recall=0.99)
    torch.cuda.synchronize()
    assert sa.sparse_attn_device_error() == 0
    Nb = -(-w.N // 64)
    mask = to_np(p.mask).astype(np.uint8)
    rng = np.random.default_rng(5)
    for h in (0, 13):
        qbs = sorted({0, Nb - 1, *rng.choice(Nb, size=6, replace=False).tolist()})
        sl = slice(h, h + 1)
        _check_against_oracle(q[:, sl].cpu(), k[:, sl].cpu(), v[:, sl].cpu(), mask[:, sl], 0.99, w.causal,
                              o[:, sl], None, qblocks=qbs, max_excused_frac=1.0)


def test_recall_argument_errors():
    q, k, v = wl.random_qkv(1, 1, 128, 64, seed=0, device=_dev())
    mask = torch.ones((1, 1, 2, 2), dtype=torch.uint8, device=_dev())
    with pytest.raises(ValueError):
        sa.sparse_attn_fwd(q, k, v, mask, -12.0, recall=0.9)
    with pytest.raises(sa.SparseAttnError):
        sa.sparse_attn_fwd(q, k, v, mask, recall=0.0)
    with pytest.raises(sa.SparseAttnError):
        sa.sparse_attn_fwd_recall(q, k, v, mask, float("nan"))
