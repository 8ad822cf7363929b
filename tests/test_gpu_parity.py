"""CUDA path (through the C ABI) against the CPU oracle, element by element.

Masks: exact except blocks whose cumulative energy lies within 1e-4 of tau.
Outputs: oracle run with the GPU's own mask, max-abs <= 2e-2 and relative
Frobenius <= 1e-2 (bf16 inputs, fp32 accumulation)."""
import math

import numpy as np
import pytest
import torch

from oracle import sparse_attn_oracle as orc
from tests.helpers import (assert_output_close, check_filter_replay, check_plan_consistency,
                           compare_masks, output_errors, to_np)

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import free_block_sparse_mean_b200 as sa
    from free_block_sparse_mean_b200 import workloads as wl


def _dev():
    return torch.device("cuda:0")


def _no_device_error():
    assert sa.sparse_attn_device_error() == 0


def _plan_and_check(q, k, tau, causal, scale=None):
    p = sa.sparse_attn_plan(q, k, tau, scale, causal, with_idx=True)
    torch.cuda.synchronize()
    mask, count, idx = to_np(p.mask), to_np(p.count), to_np(p.idx)
    check_plan_consistency(mask, count, idx)
    op = orc.plan(q.cpu(), k.cpu(), tau, scale, causal)
    rows, excused = compare_masks(mask, op, tau)
    total_rows = mask.shape[0] * mask.shape[1] * mask.shape[2]
    assert rows <= max(2, total_rows // 200), f"{rows} of {total_rows} rows differ"
    return p, mask, op


def _work_ok(p, B, H, Nb):
    """work lists every query block once, in pairs of one head; heads come in
    groups of consecutive heads whose tiles are interleaved by rank, and within a
    head the pairs' union sizes do not increase."""
    Tq = (Nb + 1) // 2
    work = to_np(p.work).astype(np.int64)[: 2 * B * H * Tq].reshape(B * H * Tq, 2)
    mask = to_np(p.mask).reshape(B * H, Nb, Nb).astype(bool)
    a, b = work[:, 0], work[:, 1]
    head = a // Nb
    assert np.all((b == -1) | (b // Nb == head))
    for bh in range(B * H):
        sel = np.nonzero(head == bh)[0]
        assert len(sel) == Tq
        ids = np.concatenate([a[sel], b[sel][b[sel] >= 0]]) - bh * Nb
        assert sorted(ids.tolist()) == list(range(Nb))
        assert (b[sel] == -1).sum() == Nb % 2
        uni = [(mask[bh, x - bh * Nb] | (mask[bh, y - bh * Nb] if y >= 0 else False)).sum()
               for x, y in zip(a[sel], b[sel])]
        if Nb <= 1024:
            assert np.all(np.diff(uni) <= 0)
    # each head's tiles fill one contiguous group of positions with the other heads of its group
    first = np.array([np.nonzero(head == bh)[0].min() for bh in range(B * H)])
    last = np.array([np.nonzero(head == bh)[0].max() for bh in range(B * H)])
    assert np.all(np.diff(first) > 0)
    for bh in range(1, B * H):
        assert first[bh] > last[bh - 1] or first[bh] == first[bh - 1] + 1


def test_pairing_reduces_union_on_small_workload():
    """On the video raster the plan's pairs must cost fewer union entries than
    the natural adjacent pairs (2t, 2t+1)."""
    w = wl.WORKLOADS["small"]
    q, k, _ = wl.generate(w, seed=0, device=_dev())
    p = sa.sparse_attn_plan(q, k, 0.95)
    torch.cuda.synchronize()
    _work_ok(p, 1, w.H, 64)
    m = to_np(p.mask).reshape(w.H, 64, 64).astype(bool)
    work = to_np(p.work).astype(np.int64).reshape(w.H * 32, 2)
    paired = sum((m[x // 64, x % 64] | m[y // 64, y % 64]).sum() for x, y in work)
    natural = sum((m[h, 2 * t] | m[h, 2 * t + 1]).sum() for h in range(w.H) for t in range(32))
    print(f"union entries: plan pairs {paired}, natural pairs {natural}, kept pairs {m.sum()}")
    assert paired < 0.8 * natural


SHAPES = [
    # B, H, N, d, causal, tau
    (1, 1, 1, 64, False, 0.9),
    (1, 2, 63, 128, False, 0.9),
    (1, 2, 64, 64, True, 0.95),
    (2, 1, 65, 128, False, 0.5),
    (1, 2, 200, 128, True, 0.9),
    (1, 3, 1000, 64, False, 0.95),
    (2, 2, 1024, 128, True, 0.99),
    (1, 2, 1500, 128, False, 1.0),
    (1, 1, 4160, 128, False, 0.8),
]


@pytest.mark.parametrize("B,H,N,d,causal,tau", SHAPES)
def test_plan_and_fwd_random(B, H, N, d, causal, tau):
    q, k, v = wl.random_qkv(B, H, N, d, seed=N + d, device=_dev(), scale_qk=2.0)
    p, mask, op = _plan_and_check(q, k, tau, causal)
    _work_ok(p, B, H, -(-N // 64))
    o = sa.sparse_attn_fwd(q, k, v, p)
    torch.cuda.synchronize()
    ref = orc.fwd(q.cpu(), k.cpu(), v.cpu(), mask, None, None, causal)
    assert_output_close(to_np(o), ref, f"fwd B{B} H{H} N{N} d{d} causal{causal}")
    _no_device_error()


@pytest.mark.parametrize("N,d,causal", [(64, 128, False), (300, 64, True), (1088, 128, False),
                                        (777, 128, True)])
def test_fwd_full_mask_is_dense(N, d, causal):
    q, k, v = wl.random_qkv(1, 2, N, d, seed=7, device=_dev())
    Nb = -(-N // 64)
    mask = torch.ones((1, 2, Nb, Nb), dtype=torch.uint8, device=_dev())
    o = sa.sparse_attn_fwd(q, k, v, mask, None, None, causal)
    torch.cuda.synchronize()
    ref = orc.attention_masked(q.cpu(), k.cpu(), v.cpu(), np.ones((1, 2, Nb, Nb), np.uint8), None, causal)
    assert_output_close(to_np(o), ref, "dense")


@pytest.mark.parametrize("N,d,causal,density", [(640, 128, False, 0.3), (1000, 64, False, 0.5),
                                                (900, 128, True, 0.4), (130, 128, False, 0.0)])
def test_fwd_random_mask(N, d, causal, density):
    """Arbitrary masks, including rows with no kept block (output 0)."""
    q, k, v = wl.random_qkv(1, 3, N, d, seed=11, device=_dev())
    Nb = -(-N // 64)
    g = torch.Generator().manual_seed(3)
    m = (torch.rand((1, 3, Nb, Nb), generator=g) < density).to(torch.uint8)
    o = sa.sparse_attn_fwd(q, k, v, m.to(_dev()), None, None, causal)
    torch.cuda.synchronize()
    ref = orc.attention_masked(q.cpu(), k.cpu(), v.cpu(), m.numpy(), None, causal)
    assert_output_close(to_np(o), ref, "random mask")
    _no_device_error()


@pytest.mark.parametrize("lam", [-12.0, -6.0, -3.0])
def test_fwd_lambda_skip(lam):
    """Key block 0 aligned with all queries, the rest weaker: later blocks fall
    below lambda. The oracle's tiled loop must give the GPU's output both on its
    own decisions (up to fp32 flips) and, exactly at the tolerance, when it
    replays the GPU's recorded decisions; each GPU decision must agree with the
    oracle's test unless that test's margin is within the fp32 border."""
    N, d = 1024, 128
    q, k, v = wl.random_qkv(1, 2, N, d, seed=5, device=_dev())
    u = torch.ones(d, device=_dev())
    q = (q.float() * 0.3 + u).to(torch.bfloat16)
    k = k.float()
    k[:, :, :64] = k[:, :, :64] * 0.3 + u
    k = k.to(torch.bfloat16)
    Nb = N // 64
    mask = torch.ones((1, 2, Nb, Nb), dtype=torch.uint8, device=_dev())
    stats = torch.zeros(4, dtype=torch.int64, device=_dev())
    dec = torch.zeros((1, 2, Nb, Nb), dtype=torch.uint8, device=_dev())
    o = sa.sparse_attn_fwd(q, k, v, mask, lam, stats=stats, decisions=dec)
    torch.cuda.synchronize()
    _no_device_error()
    ref, st = orc.attention_tiled(q.cpu(), k.cpu(), v.cpu(), to_np(mask).astype(np.uint8), lam,
                                  return_stats=True)
    assert_output_close(to_np(o), ref, f"lambda={lam}")
    st_r, flips = check_filter_replay(q.cpu(), k.cpu(), v.cpu(), to_np(mask).astype(np.uint8), o, to_np(dec),
                                      lam=lam, what=f"lambda={lam} replay")
    s = to_np(stats)
    assert s[0] == st["kept_pairs"] == st_r["kept_pairs"]
    assert s[1] == int(to_np(dec).sum())
    assert abs(int(s[1]) - st["pv_skipped"]) <= flips


def test_fwd_lambda_plain_call_equals_recorded():
    """sparse_attn_fwd and sparse_attn_fwd_decisions run the same kernel: the
    outputs and the counts are bit-identical."""
    w = wl.WORKLOADS["small"].with_(H=4)
    q, k, v = wl.generate(w, seed=2, device=_dev())
    p = sa.sparse_attn_plan(q, k, 0.95)
    s1 = torch.zeros(4, dtype=torch.int64, device=_dev())
    s2 = torch.zeros(4, dtype=torch.int64, device=_dev())
    dec = torch.zeros((1, 4, 64, 64), dtype=torch.uint8, device=_dev())
    a = sa.sparse_attn_fwd(q, k, v, p, -12.0, stats=s1)
    b = sa.sparse_attn_fwd(q, k, v, p, -12.0, stats=s2, decisions=dec)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(s1, s2)
    assert int(dec.sum()) == int(s2[1]) > 0


SMALL_POINTS = [(tau, lam) for tau in (0.90, 0.95, 0.99) for lam in (None, -12.0)]


@pytest.mark.parametrize("tau,lam", SMALL_POINTS)
def test_small_workload(tau, lam):
    """The small DiT-layer shape (H=24, d=128, N=4096), all heads, at every
    configured (tau, lambda) point: masks against the oracle's plan, outputs
    against the oracle on the GPU's mask (with lambda: replaying the GPU's
    recorded decisions, every decision checked against the oracle's test)."""
    w = wl.WORKLOADS["small"]
    q, k, v = wl.generate(w, seed=0, device=_dev())
    p, mask, op = _plan_and_check(q, k, tau, False)
    dec = torch.zeros((1, w.H, 64, 64), dtype=torch.uint8, device=_dev())
    o = sa.sparse_attn_fwd(q, k, v, p, lam, decisions=dec)
    torch.cuda.synchronize()
    _no_device_error()
    if lam is None:
        ref = orc.fwd(q.cpu(), k.cpu(), v.cpu(), mask, lam)
        assert_output_close(to_np(o), ref, f"small tau={tau} lam={lam}")
        assert int(dec.sum()) == 0
    else:
        _, flips = check_filter_replay(q.cpu(), k.cpu(), v.cpu(), mask, o, to_np(dec), lam=lam,
                                       what=f"small tau={tau} lam={lam}")
        print(f"small tau={tau} lam={lam}: {int(dec.sum())} skipped, {flips} flips within the border")
    dense = orc.attention_masked(q[:, :2].cpu(), k[:, :2].cpu(), v[:, :2].cpu(), np.ones_like(mask[:, :2]))
    max_abs, rel = output_errors(to_np(o[:, :2]), dense)
    print(f"small tau={tau} lam={lam}: sparse-vs-dense (heads 0-1) max_abs={max_abs:.3e} rel_fro={rel:.3e}, "
          f"density={mask.mean():.3f}")


def test_tiny_workload_and_sparse_vs_dense():
    w = wl.WORKLOADS["tiny"]
    q, k, v = wl.generate(w, seed=0, device=_dev())
    p, mask, op = _plan_and_check(q, k, 0.95, False)
    o = sa.sparse_attn_fwd(q, k, v, p)
    torch.cuda.synchronize()
    ref = orc.fwd(q.cpu(), k.cpu(), v.cpu(), mask)
    assert_output_close(to_np(o), ref, "tiny")
    dense = orc.attention_masked(q.cpu(), k.cpu(), v.cpu(), np.ones_like(mask))
    max_abs, rel = output_errors(to_np(o), dense)
    print(f"tiny sparse-vs-dense: max_abs={max_abs:.3e} rel_fro={rel:.3e} "
          f"density={mask.mean():.3f}")


def test_repeatable_masks():
    q, k, _ = wl.random_qkv(1, 4, 3000, 128, seed=2, device=_dev(), scale_qk=2.0)
    a = sa.sparse_attn_plan(q, k, 0.9)
    b = sa.sparse_attn_plan(q, k, 0.9)
    torch.cuda.synchronize()
    assert torch.equal(a.mask, b.mask) and torch.equal(a.count, b.count)


def test_per_head_tau_matches_oracle_and_flags_invalid_values():
    """sparse_attn_plan_heads: every head keeps its own tau's set (small DiT
    workload, tau from 0.85 to 0.99 over the heads), and a value outside (0, 1]
    keeps every block of its head and sets bit 2 of the device error word."""
    w = wl.WORKLOADS["small"]
    q, k, _ = wl.generate(w, seed=0, device=_dev())
    taus = torch.linspace(0.85, 0.99, w.H, dtype=torch.float32, device=_dev())
    p = sa.sparse_attn_plan(q, k, taus, with_idx=True)
    torch.cuda.synchronize()
    _no_device_error()
    mask, count, idx = to_np(p.mask), to_np(p.count), to_np(p.idx)
    check_plan_consistency(mask, count, idx)
    _work_ok(p, 1, w.H, 64)
    tau_np = taus.cpu().numpy().astype(np.float64)
    op = orc.plan(q.cpu(), k.cpu(), tau_np[None, :])
    rows = 0
    for h in range(w.H):
        oh = {key: op[key][:, h:h + 1] for key in ("mask", "P", "c_before", "c_after")}
        r, _ = compare_masks(mask[:, h:h + 1], oh, float(tau_np[h]))
        rows += r
    assert rows <= max(2, (w.H * 64) // 200)
    counts = count.reshape(w.H, 64).mean(-1)
    assert counts[-1] > counts[0]                      # a higher tau keeps more

    bad = taus.clone()
    bad[3] = 1.5
    bad[7] = float("nan")
    p2 = sa.sparse_attn_plan(q, k, bad)
    torch.cuda.synchronize()
    assert sa.sparse_attn_device_error() == 4
    m2 = to_np(p2.mask)
    assert np.all(m2[0, 3] == 1) and np.all(m2[0, 7] == 1)
    assert np.array_equal(m2[0, 4], mask[0, 4])


def test_end_to_end_from_pinned_host_buffers():
    """sparse_attention (the C call sparse_attn_host: host in, host out, pipelined
    over head groups on three streams) returns exactly what the device-side plan +
    forward return, for any number of groups, for a per-head tau, for the recall
    filter and for FP8 scores: heads are independent, so grouping changes nothing."""
    w = wl.WORKLOADS["small"].with_(H=6)
    q, k, v = wl.generate(w, seed=3, device=_dev())
    ref = sa.sparse_attn_fwd(q, k, v, sa.sparse_attn_plan(q, k, 0.95), -12.0)
    taus = torch.linspace(0.9, 0.97, w.H, dtype=torch.float32, device=_dev())
    ref_t = sa.sparse_attn_fwd(q, k, v, sa.sparse_attn_plan(q, k, taus), -12.0)
    ref_r = sa.sparse_attn_fwd(q, k, v, sa.sparse_attn_plan(q, k, 0.9), recall=0.95)
    p8 = sa.sparse_attn_plan(q, k, 0.95, quantize=True)
    ref_8 = sa.sparse_attn_fwd(q, k, v, p8, -12.0, qk_fp8=True)
    torch.cuda.synchronize()
    qh, kh, vh = (x.cpu().pin_memory() for x in (q, k, v))
    for chunks in (1, 4, 6):
        o = sa.sparse_attention(qh, kh, vh, 0.95, -12.0, chunks=chunks)
        assert o.device.type == "cpu" and o.is_pinned()
        assert torch.equal(o, ref.cpu()), f"chunks={chunks}"
    assert torch.equal(sa.sparse_attention(qh, kh, vh, taus, -12.0, chunks=4), ref_t.cpu())
    assert torch.equal(sa.sparse_attention(qh, kh, vh, 0.9, recall=0.95, chunks=3), ref_r.cpu())
    assert torch.equal(sa.sparse_attention(qh, kh, vh, 0.95, -12.0, chunks=2, qk_fp8=True), ref_8.cpu())
    _no_device_error()


def test_host_call_through_the_c_abi_on_one_stream():
    """sparse_attn_host called directly, both copy directions on the compute
    stream (NULL copy streams), pageable input buffers: same output."""
    import ctypes
    from free_block_sparse_mean_b200 import _lib
    lib = _lib.load()
    w = wl.WORKLOADS["small"].with_(H=3)
    q, k, v = wl.generate(w, seed=4, device=_dev())
    ref = sa.sparse_attn_fwd(q, k, v, sa.sparse_attn_plan(q, k, 0.9), None)
    torch.cuda.synchronize()
    qh, kh, vh = (x.cpu() for x in (q, k, v))
    oh = torch.empty_like(qh)
    s = _lib.SaShape(1, w.H, w.N, w.D, 64)
    nbytes = int(lib.sparse_attn_host_workspace_size(s, 2, 0))
    ws = torch.empty((nbytes,), dtype=torch.uint8, device=_dev())
    stream = torch.cuda.current_stream(_dev())
    st = lib.sparse_attn_host(ctypes.c_void_p(qh.data_ptr()), ctypes.c_void_p(kh.data_ptr()),
                              ctypes.c_void_p(vh.data_ptr()), s, 0.9, None, _lib.SA_FILTER_LAMBDA,
                              float("-inf"), w.D ** -0.5, 0, 0, ctypes.c_void_p(oh.data_ptr()),
                              ctypes.c_void_p(ws.data_ptr()), nbytes, 2, ctypes.c_void_p(stream.cuda_stream),
                              None, None)
    assert st == 0, lib.sparse_attn_status_string(st)
    stream.synchronize()
    assert torch.equal(oh, ref.cpu())
    st = lib.sparse_attn_host(ctypes.c_void_p(qh.data_ptr()), ctypes.c_void_p(kh.data_ptr()),
                              ctypes.c_void_p(vh.data_ptr()), s, 0.9, None, _lib.SA_FILTER_LAMBDA,
                              float("-inf"), w.D ** -0.5, 0, 0, ctypes.c_void_p(oh.data_ptr()),
                              ctypes.c_void_p(ws.data_ptr()), nbytes - 256, 2,
                              ctypes.c_void_p(stream.cuda_stream), None, None)
    assert st == 3                        # SA_ERR_WORKSPACE: too small, nothing enqueued
