"""Interaction clustering and the clustered attention path on the GPU (through
the C ABI) against the oracle.

The assignment is an argmin the GPU takes in fp32: a token may pick a
different cluster than the fp64 oracle only when the two clusters' distances
are within rounding of each other (checked with the oracle's own distances).
Later iterations start from the centroids the earlier ones produced, so each
iteration is checked on its own: one oracle assignment step from the GPU's
centroids must give the GPU's next assignment (near-ties excused), and
everything that follows from the GPU's assignment (the order, the centroids)
is checked exactly against that assignment. The attention itself is
compared with the oracle run on the GPU's order and mask (the pattern of the
other parity tests), and with every block kept it must equal dense attention
whatever the order."""
import numpy as np
import pytest
import torch

from oracle import sparse_attn_oracle as orc
from tests.helpers import assert_output_close, compare_masks, to_np

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import free_block_sparse_mean_b200 as sa
    from free_block_sparse_mean_b200 import workloads as wl


def _dev():
    return torch.device("cuda:0")


def _inputs(case):
    if case == "small":
        return wl.generate(wl.WORKLOADS["small"], seed=0, device=_dev(), heads=[0, 7])
    if case == "ragged64":
        q, k, v = wl.random_qkv(2, 2, 1000, 64, seed=4, device=_dev())
        drift = torch.sin(torch.arange(1000, device=_dev()) / 40.0)[None, None, :, None]
        return (q.float() * 0.5 + drift).to(torch.bfloat16), k, v
    if case in ("tiles128", "tiles64"):
        # more clusters than one centroid tile of the tensor-core assignment (64):
        # 301 clusters (five tiles, the last one partial) with d = 128, and 141
        # clusters (three tiles) over B = 2 with d = 64; CTAs of 256 tokens start in
        # every tile, so every visiting order occurs
        B, H, N, d = (1, 2, 19217, 128) if case == "tiles128" else (2, 1, 9000, 64)
        q, k, v = wl.random_qkv(B, H, N, d, seed=11, device=_dev())
        pos = torch.arange(N, device=_dev(), dtype=torch.float32)
        drift = (torch.sin(pos / 300.0)[:, None] * torch.linspace(-1.0, 1.0, d, device=_dev())[None, :]
                 + torch.cos(pos / 97.0)[:, None] * torch.linspace(1.0, -0.5, d, device=_dev())[None, :])
        drift = drift[None, None]
        return (q.float() * 0.5 + drift).to(torch.bfloat16), (k.float() * 0.5 - drift).to(torch.bfloat16), v
    raise ValueError(case)


def _check_order_and_centroids(x, res, C):
    """perm is the stable sort of the GPU's own assignment; the centroids are the
    means of its clusters (fp64 in the test)."""
    a = to_np(res.assign).astype(np.int64)
    perm = to_np(res.perm).astype(np.int64)
    np.testing.assert_array_equal(perm, np.argsort(a, axis=-1, kind="stable"))
    assert a.min() >= 0 and a.max() < C
    X = orc.as_f64(x.cpu())
    cent = to_np(res.centroids).astype(np.float64)
    B, H = a.shape[:2]
    for b in range(B):
        for h in range(H):
            for c in np.unique(a[b, h]):
                m = X[b, h, a[b, h] == c].mean(axis=0)
                np.testing.assert_allclose(cent[b, h, c], m, rtol=1e-5, atol=1e-5)


@pytest.mark.parametrize("case", ["small", "ragged64", "tiles128", "tiles64"])
@pytest.mark.parametrize("side", ["q", "k"])
def test_one_iteration_matches_the_oracle(case, side):
    q, k, _ = _inputs(case)
    x, y = (q, k) if side == "q" else (k, q)
    res = sa.sparse_attn_cluster(x, y, 1, with_centroids=True)
    torch.cuda.synchronize()
    assert sa.sparse_attn_device_error() == 0
    a_o, _, _ = orc.kmeans_interaction(x.cpu(), y.cpu(), 1)
    a_g = to_np(res.assign).astype(np.int64)
    X, Y = orc.as_f64(x.cpu()), orc.as_f64(y.cpu())
    dist = orc.interaction_distance(X, orc.block_mean_pool(X), orc.gram(Y))
    diff = np.nonzero(a_g != a_o)
    n = a_g.size
    assert len(diff[0]) <= max(2, n // 1000), f"{len(diff[0])} of {n} tokens differ"
    for b, h, t in zip(*diff):
        d = dist[b, h, t]
        gap = d[a_g[b, h, t]] - d[a_o[b, h, t]]
        assert gap <= 1e-5 * (abs(d).max() + 1.0), (b, h, t, gap)
    C = -(-x.shape[2] // 64)
    _check_order_and_centroids(x, res, C)


@pytest.mark.parametrize("case,iters", [("small", 4), ("tiles128", 3)])
@pytest.mark.parametrize("side", ["q", "k"])
def test_every_iteration_matches_an_oracle_step(case, iters, side):
    """Each Lloyd iteration on its own: from the GPU's centroids after t
    iterations, one oracle assignment step (argmin of the interaction distance,
    ties to the lowest index) must give the GPU's assignment after t + 1
    iterations, except tokens whose two distances lie within 1e-5 (relative) of
    each other; the GPU's centroids after t + 1 are the means of that assignment.
    Deterministic kernels: the first t iterations of the (t + 1)-run are the t-run."""
    q, k, _ = _inputs(case)
    x, y = (q, k) if side == "q" else (k, q)
    X, Y = orc.as_f64(x.cpu()), orc.as_f64(y.cpu())
    G = orc.gram(Y)
    C = -(-x.shape[2] // 64)
    prev = sa.sparse_attn_cluster(x, y, 1, with_centroids=True)
    for t in range(1, iters):
        nxt = sa.sparse_attn_cluster(x, y, t + 1, with_centroids=True)
        torch.cuda.synchronize()
        assert sa.sparse_attn_device_error() == 0
        cent_t = to_np(prev.centroids).astype(np.float64)
        dist = orc.interaction_distance(X, cent_t, G)
        a_o = np.argmin(dist, axis=-1)
        a_g = to_np(nxt.assign).astype(np.int64)
        diff = np.nonzero(a_g != a_o)
        for b, h, tok in zip(*diff):
            d = dist[b, h, tok]
            gap = d[a_g[b, h, tok]] - d[a_o[b, h, tok]]
            assert gap <= 1e-5 * (abs(d).max() + 1.0), (t, b, h, tok, gap)
        print(f"iteration {t + 1} ({side}): {len(diff[0])} of {a_g.size} tokens on near-ties")
        _check_order_and_centroids(x, nxt, C)
        prev = nxt


def test_zero_iterations_keep_the_blocks():
    q, k, _ = _inputs("ragged64")
    res = sa.sparse_attn_cluster(q, k, 0, with_centroids=True)
    torch.cuda.synchronize()
    N = q.shape[2]
    np.testing.assert_array_equal(to_np(res.perm), np.broadcast_to(np.arange(N), res.perm.shape))
    np.testing.assert_array_equal(to_np(res.assign), np.broadcast_to(np.arange(N) // 64, res.perm.shape))
    np.testing.assert_allclose(to_np(res.centroids), orc.block_mean_pool(orc.as_f64(q.cpu())), rtol=1e-5, atol=1e-6)


def test_permute_rows_gather_and_scatter():
    x, _, _ = wl.random_qkv(2, 3, 777, 128, seed=9, device=_dev())
    g = torch.Generator(device="cpu").manual_seed(3)
    perm = torch.stack([torch.randperm(777, generator=g) for _ in range(6)]).view(2, 3, 777).to(torch.int32)
    perm = perm.to(_dev())
    y = sa.sparse_attn_permute_rows(x, perm)
    z = sa.sparse_attn_permute_rows(y, perm, inverse=True)
    torch.cuda.synchronize()
    want = torch.gather(x, 2, perm.long()[..., None].expand(-1, -1, -1, 128))
    assert torch.equal(y, want)
    assert torch.equal(z, x)
    assert sa.sparse_attn_device_error() == 0


def test_permute_rows_range_check():
    """An entry outside 0..N-1 is caught by the kernel's own check before any
    access: that row is left alone and the range bit is set."""
    x, _, _ = wl.random_qkv(1, 1, 128, 64, seed=1, device=_dev())
    perm = torch.arange(128, dtype=torch.int32, device=_dev()).view(1, 1, 128).contiguous()
    perm[0, 0, 5] = 128
    out = torch.zeros_like(x)
    sa.sparse_attn_permute_rows(x, perm, out=out)
    torch.cuda.synchronize()
    assert sa.sparse_attn_device_error() & 2
    assert torch.equal(out[0, 0, :5], x[0, 0, :5]) and torch.all(out[0, 0, 5] == 0)


@pytest.mark.parametrize("case,iters", [("small", 2), ("ragged64", 3)])
def test_clustered_attention_with_every_block_kept_is_dense(case, iters):
    q, k, v = _inputs(case)
    o, info = sa.sparse_attention_clustered(q, k, v, 1.0, None, iters)
    torch.cuda.synchronize()
    assert sa.sparse_attn_device_error() == 0
    assert not torch.equal(info["cq"].perm[0, 0].cpu(), torch.arange(q.shape[2], dtype=torch.int32))
    B, H, N, _ = q.shape
    full = np.ones((B, H, -(-N // 64), -(-N // 64)), dtype=np.uint8)
    ref = orc.attention_masked(q.cpu(), k.cpu(), v.cpu(), full)
    assert_output_close(to_np(o), ref, f"{case} clustered, every block kept")


@pytest.mark.parametrize("tau,lam", [(0.9, None), (0.95, -12.0)])
def test_clustered_attention_matches_the_oracle_on_the_gpu_order(tau, lam):
    q, k, v = _inputs("small")
    o, info = sa.sparse_attention_clustered(q, k, v, tau, lam, 2)
    torch.cuda.synchronize()
    assert sa.sparse_attn_device_error() == 0
    pq, pk = to_np(info["cq"].perm).astype(np.int64), to_np(info["ck"].perm).astype(np.int64)
    Q, K, V = (orc.as_f64(x.cpu()) for x in (q, k, v))
    Qs = np.take_along_axis(Q, pq[..., None], axis=2)
    Ks = np.take_along_axis(K, pk[..., None], axis=2)
    Vs = np.take_along_axis(V, pk[..., None], axis=2)
    mask = to_np(info["plan"].mask)
    compare_masks(mask, orc.plan(Qs, Ks, tau), tau)
    ref, _ = orc.clustered_attention(Q, K, V, tau, lam, perms=(pq, pk))
    # the oracle's own mask may differ within the tau band; the output is checked on the GPU's mask
    Os = orc.fwd(Qs, Ks, Vs, mask, lam)
    ref_gpu_mask = np.empty_like(Os)
    np.put_along_axis(ref_gpu_mask, pq[..., None], Os, axis=2)
    assert_output_close(to_np(o), ref_gpu_mask, f"clustered tau={tau} lam={lam}")
    assert np.abs(ref - ref_gpu_mask).max() <= 5e-2


def test_cluster_argument_errors():
    q, k, _ = _inputs("ragged64")
    with pytest.raises(sa.SparseAttnError):
        sa.sparse_attn_cluster(q, k, 65)
    with pytest.raises(sa.SparseAttnError):
        sa.sparse_attn_cluster(q, k, -1)
    with pytest.raises(ValueError):
        sa.sparse_attn_permute_rows(q, torch.zeros(q.shape[:3], dtype=torch.int64, device=_dev()))
