"""Pins of the CPU oracle to facts outside itself (no GPU).

Each test checks the oracle against something it does not compute itself: a
closed form, a library routine, brute force on tiny inputs, hand-worked cases, or
an invariant of the definition; chosen so that a dropped term, a wrong index, a
transposed operand or a wrong tie rule fails at least one of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import softmax as scipy_softmax

from oracle import sparse_attn_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


# ------------------------------------------------------------------ pooling + logits

@pytest.mark.parametrize("N", [1, 63, 64, 65, 200, 256])
def test_pool_is_block_average_of_token_logits(N):
    """Bilinearity: scale * <mean Q_blk i, mean K_blk j> equals the mean of the
    n_i x n_j block of full-resolution scaled logits (ragged tail included)."""
    r = _rng(N)
    d = 8
    Q = r.standard_normal((2, 3, N, d))
    K = r.standard_normal((2, 3, N, d))
    scale = 0.37
    L = orc.pooled_logits(orc.block_mean_pool(Q), orc.block_mean_pool(K), scale, False)
    S = scale * np.einsum("bhnd,bhmd->bhnm", Q, K)
    starts = np.arange(0, N, 64)
    Sr = np.add.reduceat(np.add.reduceat(S, starts, axis=2), starts, axis=3)
    sizes = np.minimum(starts + 64, N) - starts
    ref = Sr / (sizes[:, None] * sizes[None, :])
    np.testing.assert_allclose(L, ref, rtol=1e-12, atol=1e-12)


def test_pool_closed_form_row_index():
    """Rows equal to their token index: block mean = (first + last) / 2, tail too."""
    N = 150
    X = np.repeat(np.arange(N, dtype=np.float64)[:, None], 3, axis=1)[None, None]
    P = orc.block_mean_pool(X)
    expect = [(0 + 63) / 2, (64 + 127) / 2, (128 + 149) / 2]
    np.testing.assert_array_equal(P[0, 0, :, 0], expect)


def test_causal_pooled_logits_exclude_later_blocks():
    r = _rng(1)
    Qp = r.standard_normal((1, 1, 5, 4))
    L = orc.pooled_logits(Qp, Qp, 1.0, True)
    assert np.all(np.isneginf(L[0, 0][np.triu_indices(5, 1)]))
    assert np.all(np.isfinite(L[0, 0][np.tril_indices(5)]))


# ------------------------------------------------------------------ softmax

def test_pooled_softmax_matches_library():
    r = _rng(2)
    L = 3.0 * r.standard_normal((2, 3, 7, 7))
    np.testing.assert_allclose(orc.pooled_softmax(L), scipy_softmax(L, axis=-1), rtol=1e-13)
    Lc = orc.pooled_logits(r.standard_normal((1, 1, 6, 3)), r.standard_normal((1, 1, 6, 3)), 1.0, True)
    P = orc.pooled_softmax(Lc)
    np.testing.assert_allclose(P.sum(-1), 1.0, rtol=1e-14)
    assert np.all(P[0, 0][np.triu_indices(6, 1)] == 0.0)


# ------------------------------------------------------------------ selection

def test_select_golden_hand_worked():
    with open(os.path.join(GOLDEN, "select_cases.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        p = np.array(c["p"], dtype=np.float64)[None]
        mask, count, idx, cb, ca = orc.cumulative_energy_select(p, c["tau"])
        assert int(count[0]) == c["count"], c
        assert list(idx[0, : c["count"]]) == c["idx"], c
        assert list(np.nonzero(mask[0])[0]) == c["idx"], c
        assert np.all(idx[0, c["count"]:] == -1)
        # the running sums in sorted order are the hand-worked ones
        order = np.argsort(-p[0], kind="stable")
        np.testing.assert_array_equal(ca[0, order], c["running"])


def test_select_end_to_end_constructed_inputs():
    """Q rows all (1,0); K block j rows all (ln p_j, 0); scale 1: the pooled map of
    every query block is p exactly, so the plan must keep the hand-worked set
    {1, 2, 3} at tau = 0.9 for p = (1/16, 8/16, 2/16, 5/16). A ragged last block
    (8 tokens) must not change that."""
    p = np.array([1 / 16, 8 / 16, 2 / 16, 5 / 16])
    for N in (256, 200):
        Q = np.zeros((1, 1, N, 2)); Q[..., 0] = 1.0
        K = np.zeros((1, 1, N, 2))
        for j in range(4):
            K[0, 0, j * 64:min(N, (j + 1) * 64), 0] = math.log(p[j])
        out = orc.plan(Q, K, 0.9, scale=1.0)
        np.testing.assert_allclose(out["P"][0, 0], np.tile(p, (4, 1)), rtol=1e-14)
        assert np.all(out["mask"][0, 0] == np.array([0, 1, 1, 1]))
        assert np.all(out["count"][0, 0] == 3)


@pytest.mark.parametrize("Nb", [1, 2, 3, 5, 8, 10])
def test_select_minimal_cardinality_brute_force(Nb):
    """The kept count equals the smallest size of ANY subset reaching tau of the
    row total (enumerated), and the kept set has the largest sum among sets of
    that size."""
    r = _rng(Nb)
    for trial in range(25):
        p = r.dirichlet(np.full(Nb, 0.6))
        tau = float(r.uniform(0.3, 0.999))
        mask, count, idx, _, _ = orc.cumulative_energy_select(p[None], tau)
        best = None
        best_sum_at_k = {}
        for k in range(1, Nb + 1):
            sums = [sum(p[list(s)]) for s in itertools.combinations(range(Nb), k)]
            best_sum_at_k[k] = max(sums)
            if best is None and best_sum_at_k[k] >= tau * p.sum() - 1e-15:
                best = k
        assert int(count[0]) == best
        kept_sum = p[mask[0].astype(bool)].sum()
        assert kept_sum >= tau * p.sum() - 1e-15
        assert abs(kept_sum - best_sum_at_k[best]) < 1e-12


def test_select_invariants_random_rows():
    r = _rng(7)
    P = orc.pooled_softmax(2.5 * r.standard_normal((3, 4, 40, 40)))
    for tau in (0.5, 0.9, 0.95, 0.99):
        mask, count, idx, cb, ca = orc.cumulative_energy_select(P, tau)
        kept = mask.astype(bool)
        e = np.where(kept, P, 0).sum(-1)
        assert np.all(e >= tau - 1e-12)                       # recall reached
        smallest = np.where(kept, P, np.inf).min(-1)
        assert np.all(e - smallest < tau + 1e-12)             # minimal
        assert np.array_equal(kept.sum(-1), count)
        # idx ascending, consistent with the mask
        for flat in range(0, 3 * 4 * 40, 37):
            b, h, i = np.unravel_index(flat, count.shape)
            row = idx[b, h, i, : count[b, h, i]]
            assert np.all(np.diff(row) > 0)
            assert np.array_equal(row, np.nonzero(mask[b, h, i])[0])


def test_select_special_cases():
    Nb = 12
    # tau = 1 keeps every block with positive energy
    r = _rng(3)
    p = r.dirichlet(np.ones(Nb))
    mask, count, *_ = orc.cumulative_energy_select(p[None], 1.0)
    assert count[0] == Nb
    # one-hot row keeps one block
    oh = np.zeros(Nb); oh[5] = 1.0
    mask, count, idx, *_ = orc.cumulative_energy_select(oh[None], 0.9)
    assert count[0] == 1 and idx[0, 0] == 5
    # uniform row: tau = (k - 1/2)/Nb keeps k blocks, the lowest indices (ties)
    u = np.full(Nb, 1.0 / Nb)
    for k in range(1, Nb + 1):
        mask, count, idx, *_ = orc.cumulative_energy_select(u[None], (k - 0.5) / Nb)
        assert count[0] == k
        assert list(idx[0, :k]) == list(range(k))


def test_select_per_head_tau():
    """One tau per (batch, head) applies to every row of that head: each row's kept
    count is the smallest size of any subset reaching its head's tau (brute force),
    the kept energy reaches it, tau = 1 keeps every block, and an [H] tau
    broadcasts over the batch."""
    r = _rng(11)
    B, H, Nb = 2, 3, 8
    P = orc.pooled_softmax(2.0 * r.standard_normal((B, H, Nb, Nb)))
    taus = np.array([[1.0, 0.5, 0.9], [0.7, 0.99, 0.3]])
    mask, count, idx, cb, ca = orc.cumulative_energy_select(P, taus)
    for b in range(B):
        for h in range(H):
            t = taus[b, h]
            for i in range(Nb):
                p = P[b, h, i]
                k_min = next(k for k in range(1, Nb + 1)
                             if max(sum(p[list(c)]) for c in itertools.combinations(range(Nb), k))
                             >= t * p.sum() - 1e-15)
                assert count[b, h, i] == k_min
                assert p[mask[b, h, i].astype(bool)].sum() >= t * p.sum() - 1e-15
            if t == 1.0:
                assert np.all(mask[b, h] == 1)
    m_h, c_h, *_ = orc.cumulative_energy_select(P, taus[0])
    m_bh, c_bh, *_ = orc.cumulative_energy_select(P, np.broadcast_to(taus[0], (B, H)))
    assert np.array_equal(m_h, m_bh) and np.array_equal(c_h, c_bh)


# ------------------------------------------------------------------ attention

def _sdpa64(Q, K, V, causal, scale):
    q, k, v = (torch.from_numpy(np.ascontiguousarray(x)) for x in (Q, K, V))
    return torch.nn.functional.scaled_dot_product_attention(
        q, k, v, is_causal=causal, scale=scale).numpy()


@pytest.mark.parametrize("N,causal", [(64, False), (200, False), (130, True), (256, True), (1, False)])
def test_full_mask_equals_library_dense_attention(N, causal):
    """tau = 1 through the whole oracle (plan + fwd, lambda off) reproduces the
    library's dense fp64 attention."""
    r = _rng(N)
    d = 16
    Q = r.standard_normal((2, 2, N, d))
    K = r.standard_normal((2, 2, N, d))
    V = r.standard_normal((2, 2, N, d))
    scale = 1 / math.sqrt(d)
    pl = orc.plan(Q, K, 1.0, scale, causal)
    Nb = orc.n_blocks(N)
    full = np.ones((Nb, Nb), dtype=np.uint8)
    if causal:
        full = np.tril(full)
    assert np.array_equal(pl["mask"], np.broadcast_to(full, pl["mask"].shape))
    O = orc.fwd(Q, K, V, pl["mask"], None, scale, causal)
    np.testing.assert_allclose(O, _sdpa64(Q, K, V, causal, scale), rtol=1e-11, atol=1e-12)
    O2 = orc.attention_tiled(Q, K, V, pl["mask"], -math.inf, scale, causal)
    np.testing.assert_allclose(O2, _sdpa64(Q, K, V, causal, scale), rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("N,causal", [(300, False), (257, True)])
def test_tiled_recurrence_equals_masked_softmax(N, causal):
    """With lambda = -inf the tiled online-softmax loop equals the direct masked
    softmax on a random block mask (pins the recurrence: rescale, running sum)."""
    r = _rng(N + 1)
    d = 8
    Q, K, V = (r.standard_normal((1, 2, N, d)) * 2 for _ in range(3))
    Nb = orc.n_blocks(N)
    mask = (r.random((1, 2, Nb, Nb)) < 0.5).astype(np.uint8)
    mask[..., np.arange(Nb), np.arange(Nb)] = 1
    a = orc.attention_masked(Q, K, V, mask, None, causal)
    b = orc.attention_tiled(Q, K, V, mask, -math.inf, None, causal)
    np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-13)


def _two_block_case(first_logit, second_logit):
    N, d = 128, 2
    Q = np.zeros((1, 1, N, d)); Q[..., 0] = 1.0
    K = np.zeros((1, 1, N, d))
    K[0, 0, :64, 0] = first_logit
    K[0, 0, 64:, 0] = second_logit
    V = np.zeros((1, 1, N, d))
    V[0, 0, :64, 0] = 1.0
    V[0, 0, 64:, 1] = 1.0
    mask = np.ones((1, 1, 2, 2), dtype=np.uint8)
    return Q, K, V, mask


def test_lambda_skip_closed_form():
    """Scores 0 on key block 0 and -20 on key block 1 (visited second). Off or
    lam = -25: O = (1, e^-20)/(1 + e^-20). lam = -12: P.V of block 1 is skipped
    but it stays in the running sum: O = (1, 0)/(1 + e^-20)."""
    Q, K, V, mask = _two_block_case(0.0, -20.0)
    t = math.exp(-20.0)
    O_off = orc.fwd(Q, K, V, mask, None, 1.0)
    O_25, st25 = orc.attention_tiled(Q, K, V, mask, -25.0, 1.0, return_stats=True)
    O_12, st12 = orc.attention_tiled(Q, K, V, mask, -12.0, 1.0, return_stats=True)
    np.testing.assert_allclose(O_off[0, 0], np.tile([1 / (1 + t), t / (1 + t)], (128, 1)), rtol=1e-14)
    np.testing.assert_allclose(O_25, O_off, rtol=1e-14, atol=0)
    np.testing.assert_allclose(O_12[0, 0], np.tile([1 / (1 + t), 0.0], (128, 1)), rtol=1e-14, atol=0)
    assert (st12["kept_pairs"], st12["pv_skipped"]) == (4, 2) and st25["pv_skipped"] == 0
    # margins: lam - (rowmax - m) of the second block is -12 + 20 = 8 (skip); the
    # first block of a row is never skipped (margin -inf)
    margins = sorted(mg for *_, mg in st12["decisions"])
    assert margins[:2] == [-math.inf, -math.inf]
    np.testing.assert_allclose(margins[2:], [8.0, 8.0], rtol=1e-14)


def test_lambda_first_block_never_skipped_and_order_matters():
    """Block 0 at -20, block 1 at 0: the low block comes first (running max -inf,
    never skipped) and block 1 raises the max; nothing is skipped at any lam."""
    Q, K, V, mask = _two_block_case(-20.0, 0.0)
    O_off = orc.fwd(Q, K, V, mask, None, 1.0)
    O_lam, st = orc.attention_tiled(Q, K, V, mask, -1.0, 1.0, return_stats=True)
    assert st["pv_skipped"] == 0
    np.testing.assert_allclose(O_lam, O_off, rtol=1e-14)


def test_lambda_error_bounded_by_skipped_mass():
    """Skipping only P.V leaves l unchanged, so per row
    O_lam - O_off = -(sum of skipped P V) / l, whose size is at most
    (skipped P mass / l) * max|V|; every skipped entry is below e^lam times the
    running max's weight (1), and l >= 1. Inputs: key block 0 aligned with
    every query, the other blocks pure noise, so later blocks fall below lam."""
    r = _rng(11)
    N, d = 512, 16
    u = np.ones(d)
    Q = 2.0 * u + 0.3 * r.standard_normal((1, 2, N, d))
    K = r.standard_normal((1, 2, N, d))
    K[:, :, :64] = 2.0 * u + 0.3 * r.standard_normal((1, 2, 64, d))
    V = r.standard_normal((1, 2, N, d))
    Nb = orc.n_blocks(N)
    mask = np.ones((1, 2, Nb, Nb), dtype=np.uint8)
    lam = -8.0
    O_off = orc.attention_masked(Q, K, V, mask)
    O_lam, st = orc.attention_tiled(Q, K, V, mask, lam, return_stats=True)
    assert st["pv_skipped"] == 2 * Nb * (Nb - 1)          # every non-aligned block
    assert np.abs(O_lam - O_off).max() > 0
    bound = np.abs(V).max() * (Nb - 1) * 64 * math.exp(lam)
    assert np.abs(O_lam - O_off).max() <= bound


# ---------------------------------------------------------------- in-operator recall filter
@pytest.mark.parametrize("c,recall,skipped", [(5.0, 0.99, True), (5.0, 0.995, False),
                                               (1.0, 0.7, True), (1.0, 0.75, False)])
def test_recall_skip_closed_form(c, recall, skipped):
    """Scores 0 on key block 0 and -c on key block 1 (visited second); t = e^-c.
    Block 1 carries the energy fraction t / (1 + t) of the row, so it is skipped
    exactly when t / (1 + t) <= 1 - recall: recall <= 1 / (1 + t), which is 0.99331
    for c = 5 and 0.7311 for c = 1 (where 1 - recall = 0.3 lies between
    t / (1 + t) = 0.269 and t = 0.368: the block's own energy counts in the sum).
    Skipped: O = (1, 0) / (1 + t) (l keeps the block); kept: O = (1, t) / (1 + t)."""
    Q, K, V, mask = _two_block_case(0.0, -c)
    t = math.exp(-c)
    O, st = orc.attention_recall(Q, K, V, mask, recall, 1.0, return_stats=True)
    want = [1 / (1 + t), 0.0 if skipped else t / (1 + t)]
    np.testing.assert_allclose(O[0, 0], np.tile(want, (128, 1)), rtol=1e-14, atol=0)
    assert st["kept_pairs"] == 4 and st["pv_skipped"] == (2 if skipped else 0)
    np.testing.assert_allclose(st["recall_rows"][0, 0], 1 / (1 + t) if skipped else 1.0, rtol=1e-14)


def test_recall_first_block_never_skipped_and_old_sums_rescaled():
    """Block 0 at -20 then block 1 at 0: block 0 comes first (nothing to compare
    with) and block 1 holds almost all of the energy once the old sum is rescaled
    to the new max (e^-20 * 64 against 64), so nothing is skipped even at
    recall = 0.5. Without the rescale the first block's sum would hide block 1."""
    Q, K, V, mask = _two_block_case(-20.0, 0.0)
    O_off = orc.fwd(Q, K, V, mask, None, 1.0)
    O, st = orc.attention_recall(Q, K, V, mask, 0.5, 1.0, return_stats=True)
    assert st["pv_skipped"] == 0
    np.testing.assert_allclose(O, O_off, rtol=1e-14)


def test_recall_sums_rescaled_when_the_max_rises():
    """Four key blocks with scores 0, -5, 3, -2 (t = e^-5), recall 0.99, visited in
    that order. Block 1 holds t / (1 + t) = 0.0067 <= 0.01 of the energy: skipped.
    Block 2 raises the max by 3 and holds most of the energy: kept. Block 3 (e^-5
    against the new max): skipped-so-far t e^-3 plus its own t is 0.00707, within
    0.01 of the sum e^-3 (1 + t) + 1 + t = 1.0568: skipped. Had the skipped sum
    not been rescaled to the new max (t + t = 0.0135) it would be kept.
    O = (e^-3, 0, 1, 0) / (e^-3 + e^-8 + 1 + e^-5)."""
    N, d = 256, 4
    Q = np.zeros((1, 1, N, d)); Q[..., 0] = 1.0
    K = np.zeros((1, 1, N, d))
    V = np.zeros((1, 1, N, d))
    for j, sc in enumerate([0.0, -5.0, 3.0, -2.0]):
        K[0, 0, 64 * j:64 * j + 64, 0] = sc
        V[0, 0, 64 * j:64 * j + 64, j] = 1.0
    mask = np.ones((1, 1, 4, 4), dtype=np.uint8)
    O, st = orc.attention_recall(Q, K, V, mask, 0.99, 1.0, return_stats=True)
    z = math.exp(-3) + math.exp(-8) + 1 + math.exp(-5)
    np.testing.assert_allclose(O[0, 0], np.tile([math.exp(-3) / z, 0, 1 / z, 0], (N, 1)), rtol=1e-13, atol=0)
    assert [x[4] for x in st["decisions"][:4]] == [False, True, False, True]
    np.testing.assert_allclose(st["recall_rows"][0, 0], (math.exp(-3) + 1) / z, rtol=1e-13)


def test_recall_block_that_raises_the_max_can_be_skipped():
    """Recall 0.95; key block 0 at score 0, block 1 at -5 (t = e^-5), block 2 one
    key at +1 and 63 at -50. Block 1: t / (1 + t) <= 0.05, skipped. Block 2 raises
    the max by 1 but holds one key's worth of energy: against the new max the
    skipped sum is 64 t e^-1 = 0.1586, plus its own 1 gives 1.1586 <= 0.05 *
    (64 (1 + t) e^-1 + 1) = 1.2351: skipped (the skipped sum unrescaled, 1.4312,
    would keep it). O = (64 e^-1, 0, 0) / (64 e^-1 + 64 e^-6 + 1 + 63 e^-51)."""
    N, d = 192, 3
    Q = np.zeros((1, 1, N, d)); Q[..., 0] = 1.0
    K = np.zeros((1, 1, N, d))
    V = np.zeros((1, 1, N, d))
    K[0, 0, 64:128, 0] = -5.0
    K[0, 0, 128:, 0] = -50.0
    K[0, 0, 128, 0] = 1.0
    for j in range(3):
        V[0, 0, 64 * j:64 * j + 64, j] = 1.0
    mask = np.ones((1, 1, 3, 3), dtype=np.uint8)
    O, st = orc.attention_recall(Q, K, V, mask, 0.95, 1.0, return_stats=True)
    z = 64 * math.exp(-1) + 64 * math.exp(-6) + 1 + 63 * math.exp(-51)
    np.testing.assert_allclose(O[0, 0], np.tile([64 * math.exp(-1) / z, 0, 0], (N, 1)), rtol=1e-13, atol=0)
    assert [x[4] for x in st["decisions"][:3]] == [False, True, True]


def _recall_case(seed, N, d, causal, aligned=0):
    """Key block `aligned` aligned with every query, the rest noise of varied
    strength per block, a random block mask with the diagonal and the aligned
    block kept. With aligned > 0 the running max rises midway through the row."""
    r = _rng(seed)
    u = np.ones(d)
    Nb = orc.n_blocks(N)
    Q = 1.5 * u + 0.5 * r.standard_normal((1, 2, N, d))
    K = r.standard_normal((1, 2, N, d))
    K *= np.repeat(r.uniform(0.05, 1.5, size=(1, 2, Nb, 1)), 64, axis=2)[:, :, :N]
    a = slice(64 * aligned, 64 * aligned + 64)
    K[:, :, a] = 1.5 * u + 0.5 * r.standard_normal((1, 2, 64, d))
    V = r.standard_normal((1, 2, N, d))
    mask = (r.random((1, 2, Nb, Nb)) < 0.6).astype(np.uint8)
    mask[..., np.arange(Nb), np.arange(Nb)] = 1
    mask[..., aligned] = 1
    return Q, K, V, mask


@pytest.mark.parametrize("N,causal,recall,aligned", [(512, False, 0.99, 0), (449, True, 0.95, 0),
                                                     (320, False, 0.9, 0), (640, False, 0.97, 5),
                                                     (577, True, 0.9, 3)])
def test_recall_decisions_and_output_brute_force(N, causal, recall, aligned):
    """Brute force without a running max: every row's block energies are taken
    against one fixed reference (the row's largest visible score), and the sums
    of earlier blocks are plain sums. Block j of query block i is skipped iff for
    every row that sees it, skipped-so-far + E_j <= (1 - recall) * (seen-so-far
    + E_j). The output is the unskipped blocks' weighted V over the energy of all
    visited blocks. The oracle's decisions and output must agree."""
    d = 16
    Q, K, V, mask = _recall_case(N + int(causal), N, d, causal, aligned)
    scale = 1.0 / math.sqrt(d)
    O, st = orc.attention_recall(Q, K, V, mask, recall, None, causal, return_stats=True)
    dec = {(b, h, i, j): (sk, mg) for b, h, i, j, sk, mg in st["decisions"]}
    Nb = orc.n_blocks(N)
    n_skip = 0
    for h in range(2):
        for i in range(Nb):
            s, e = i * 64, min(N, i * 64 + 64)
            S = scale * Q[0, h, s:e] @ K[0, h].T
            vis = np.repeat(mask[0, h, i].astype(bool), 64)[:N][None, :].repeat(e - s, 0)
            if causal:
                vis &= np.arange(N)[None, :] <= np.arange(s, e)[:, None]
            S = np.where(vis, S, -np.inf)
            M = S.max(axis=1)
            W = np.exp(S - M[:, None])
            seen = np.zeros(e - s)
            skipped = np.zeros(e - s)
            num = np.zeros((e - s, d))
            for j in np.nonzero(mask[0, h, i])[0]:
                cols = slice(j * 64, min(N, j * 64 + 64))
                sees = vis[:, cols].any(axis=1)
                if not sees.any():
                    continue
                E = W[:, cols].sum(axis=1)
                ok = skipped + E <= (1 - recall) * (seen + E)
                skip = bool(ok[sees].all())
                got, margin = dec[(0, h, i, int(j))]
                if abs(margin) > 1e-9:
                    assert got == skip, (h, i, j)
                skip = got
                seen += E
                if skip:
                    skipped += E
                    n_skip += 1
                else:
                    num += W[:, cols] @ V[0, h, cols]
            np.testing.assert_allclose(O[0, h, s:e], num / seen[:, None], rtol=1e-10, atol=1e-12)
            assert np.all(skipped <= (1 - recall) * seen * (1 + 1e-12))
    assert n_skip == st["pv_skipped"] and n_skip > 0
    assert np.all(st["recall_rows"][np.isfinite(st["recall_rows"])] >= recall - 1e-12)


@pytest.mark.parametrize("recall", [0.9, 0.99])
def test_recall_error_bounded_by_budget(recall):
    """The skipped blocks stay in l, so per row O_recall - O_off = -(skipped
    weighted V) / l, at most (skipped energy / l) * max|V| <= (1 - recall) * max|V|
    in every element; recall = 1 skips nothing and is the masked attention."""
    Q, K, V, mask = _recall_case(3, 384, 8, False)
    O_off = orc.attention_masked(Q, K, V, mask)
    O, st = orc.attention_recall(Q, K, V, mask, recall, return_stats=True)
    assert st["pv_skipped"] > 0
    assert np.abs(O - O_off).max() <= (1 - recall) * np.abs(V).max() * (1 + 1e-12)
    O1, st1 = orc.attention_recall(Q, K, V, mask, 1.0, return_stats=True)
    assert st1["pv_skipped"] == 0
    np.testing.assert_allclose(O1, O_off, rtol=1e-11, atol=1e-13)


def test_row_without_visible_key_is_zero():
    r = _rng(5)
    Q, K, V = (r.standard_normal((1, 1, 128, 4)) for _ in range(3))
    mask = np.zeros((1, 1, 2, 2), dtype=np.uint8)
    mask[0, 0, 1, 1] = 1
    O = orc.attention_masked(Q, K, V, mask)
    assert np.all(O[0, 0, :64] == 0)
    O2 = orc.attention_tiled(Q, K, V, mask, -5.0)
    assert np.all(O2[0, 0, :64] == 0)
    np.testing.assert_allclose(O[0, 0, 64:], O2[0, 0, 64:], rtol=1e-12)


def test_bf16_inputs_are_upcast_exactly():
    x = torch.randn(3, 5).to(torch.bfloat16)
    y = orc.as_f64(x)
    assert y.dtype == np.float64
    assert np.array_equal(y, x.float().numpy().astype(np.float64))


# ---------------------------------------------------------------- FP8 E4M3 quantization
def test_round_e4m3_matches_the_format_and_torch():
    """Hand values from the E4M3 definition (3 mantissa bits, ties to even,
    subnormal spacing 2^-9, largest 448, saturating), then torch's own
    float8_e4m3fn cast on 200k values spread over every binade."""
    hand = {0.3: 0.3125, 1.0625: 1.0, 1.1875: 1.25, 2.0 ** -10: 0.0, 3 * 2.0 ** -10: 2.0 ** -8,
            2.0 ** -9: 2.0 ** -9, 0.875 * 2.0 ** -6: 0.875 * 2.0 ** -6, 240.0: 240.0, 232.0: 224.0,
            448.0: 448.0, 460.0: 448.0, 1.0e4: 448.0, -0.3: -0.3125, 0.0: 0.0}
    for x, want in hand.items():
        assert orc.round_e4m3(x) == want, x
    r = _rng(11)
    x = np.sign(r.standard_normal(200000)) * np.exp2(r.uniform(-14.0, 8.85, 200000))   # |x| < 462
    t = torch.tensor(x, dtype=torch.float64).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(orc.round_e4m3(x), t)


def test_quantize_blocks_e4m3_scales_and_error_bound():
    r = _rng(12)
    X = r.standard_normal((1, 2, 200, 16)) * np.array([1.0, 30.0])[None, :, None, None]
    X[0, 1, 64:128] = 0.0                                    # an all-zero block
    codes, scales = orc.quantize_blocks_e4m3(X)
    assert scales.shape == (1, 2, 4)
    assert scales[0, 1, 1] == 1.0 and np.all(codes[0, 1, 64:128] == 0)
    for h in range(2):
        for i in range(4):
            blk = slice(64 * i, min(200, 64 * i + 64))
            c = codes[0, h, blk]
            if scales[0, h, i] != 1.0 or np.any(c):
                assert np.abs(c).max() == 448.0                  # the block's absmax maps to 448
            assert np.array_equal(c, orc.round_e4m3(c))          # every code is an E4M3 value
            deq = c * scales[0, h, i]
            err = np.abs(deq - X[0, h, blk])
            # half a step of the code's binade (relative 2^-4), or of the subnormal spacing
            bound = np.maximum(np.abs(X[0, h, blk]) * 2.0 ** -4, scales[0, h, i] * 2.0 ** -10) * 1.0001
            assert np.all(err <= bound)


def test_fwd_fp8qk_is_fwd_when_q_and_k_are_representable():
    """Inputs that are E4M3 values times a power of two, each block holding a 448,
    quantize exactly, so the quantized forward equals the plain one; on generic
    inputs it stays within the quantization error."""
    r = _rng(13)
    grid = orc.round_e4m3(r.uniform(-448, 448, (1, 2, 192, 8)))
    grid[:, :, ::64, 0] = 448.0
    Q, K = grid * 2.0 ** -7, orc.round_e4m3(r.uniform(-448, 448, (1, 2, 192, 8)))
    K[:, :, ::64, 0] = 448.0
    K = K * 2.0 ** -8
    V = r.standard_normal((1, 2, 192, 8))
    mask = (r.uniform(size=(1, 2, 3, 3)) < 0.7).astype(np.uint8)
    mask[..., 0, 0] = 1
    for lam in (None, -2.0):
        np.testing.assert_array_equal(orc.fwd_fp8qk(Q, K, V, mask, lam), orc.fwd(Q, K, V, mask, lam))
    Qg, Kg = r.standard_normal((1, 2, 192, 8)), r.standard_normal((1, 2, 192, 8))
    a, b = orc.fwd_fp8qk(Qg, Kg, V, mask), orc.fwd(Qg, Kg, V, mask)
    assert 0 < np.abs(a - b).max() < 0.1


# ---------------------------------------------------------------- interaction clustering
def test_interaction_distance_is_the_summed_squared_score_change():
    """Replacing x by c changes its score with every token y of the other side by
    (x - c).y; the quadratic form under the other side's Gram matrix is the sum
    of the squares of those changes (brute force over y)."""
    r = _rng(21)
    X, C, Y = r.standard_normal((1, 1, 7, 5)), r.standard_normal((1, 1, 3, 5)), r.standard_normal((1, 1, 11, 5))
    D = orc.interaction_distance(X, C, orc.gram(Y))
    for n in range(7):
        for m in range(3):
            brute = sum(float(np.dot(X[0, 0, n] - C[0, 0, m], Y[0, 0, t])) ** 2 for t in range(11))
            assert D[0, 0, n, m] == pytest.approx(brute, rel=1e-12)


def test_kmeans_metric_comes_from_the_other_side():
    """Keys all along e1 (G_K = 64 e1 e1^T): a query differing from a centroid
    only in e2 is at distance 0 from it, whatever the Euclidean distance. Query
    block 0 holds x = (0, 10) and 63 copies of (0, 0); block 1 holds (0.9, 10)
    x 64. Under the key metric x joins block 0's cluster (distance 0 against
    0.81 * 64 to the other); under the Euclidean or the query-side metric it
    would join block 1's."""
    d = 2
    Q = np.zeros((1, 1, 128, d))
    Q[0, 0, 0] = [0.0, 10.0]
    Q[0, 0, 64:] = [0.9, 10.0]
    K = np.zeros((1, 1, 128, d)); K[..., 0] = 1.0
    a, c, _ = orc.kmeans_interaction(Q, K, 1)
    assert a[0, 0, 0] == 0 and np.all(a[0, 0, 1:64] == 0) and np.all(a[0, 0, 64:] == 1)
    a_wrong, _, _ = orc.kmeans_interaction(Q, Q, 1)       # query-side metric
    assert a_wrong[0, 0, 0] == 1


def test_kmeans_separates_two_interleaved_groups_in_one_iteration():
    """Tokens equal to a or b (a - b not in the null space of G): block 0 holds 48
    a and 16 b, block 1 16 a and 48 b, interleaved. The initial centroids are
    (3a + b)/4 and (a + 3b)/4, so one iteration sends every a to cluster 0 and
    every b to cluster 1, and the centroids become a and b exactly. The order puts
    the a tokens first, each group in token order."""
    r = _rng(5)
    d = 6
    a_vec, b_vec = r.standard_normal(d), r.standard_normal(d)
    is_a = np.zeros(128, dtype=bool)
    is_a[np.arange(0, 64)[np.arange(64) % 4 != 3]] = True      # 48 of block 0
    is_a[64 + np.arange(0, 64, 4)] = True                       # 16 of block 1
    X = np.where(is_a[:, None], a_vec, b_vec)[None, None]
    Y = r.standard_normal((1, 1, 128, d))
    a, c, obj = orc.kmeans_interaction(X, Y, 1)
    np.testing.assert_array_equal(a[0, 0], np.where(is_a, 0, 1))
    np.testing.assert_allclose(c[0, 0], np.stack([a_vec, b_vec]), rtol=1e-14, atol=1e-14)
    perm = orc.cluster_permutation(a)[0, 0]
    np.testing.assert_array_equal(perm, np.concatenate([np.nonzero(is_a)[0], np.nonzero(~is_a)[0]]))
    assert obj[1] == pytest.approx(0.0, abs=1e-9) and obj[0] > 0


@pytest.mark.parametrize("N", [300, 256])
def test_kmeans_objective_never_increases(N):
    """Lloyd iterations under a positive semi-definite metric: the assignment step
    and the mean step (the minimiser of the cluster's summed quadratic form) can
    only lower the objective."""
    r = _rng(N)
    X, Y = r.standard_normal((1, 2, N, 8)) + np.linspace(0, 3, N)[None, None, :, None], r.standard_normal((1, 2, N, 8))
    _, _, obj = orc.kmeans_interaction(X, Y, 5)
    assert all(b <= a * (1 + 1e-12) for a, b in zip(obj, obj[1:]))
    assert obj[-1] < obj[0]


def test_zero_iterations_is_block_pooling():
    r = _rng(8)
    Q, K, V = (r.standard_normal((1, 2, 200, 8)) for _ in range(3))
    a, c, _ = orc.kmeans_interaction(Q, K, 0)
    np.testing.assert_array_equal(a[0, 1], np.arange(200) // 64)
    np.testing.assert_allclose(c, orc.block_mean_pool(Q), rtol=0, atol=0)
    O, info = orc.clustered_attention(Q, K, V, 0.9, None, 0)
    p = orc.plan(Q, K, 0.9)
    np.testing.assert_allclose(O, orc.fwd(Q, K, V, p["mask"]), rtol=1e-13, atol=1e-14)


@pytest.mark.parametrize("iters", [1, 3])
def test_clustered_attention_with_every_block_kept_is_dense(iters):
    """Attention is invariant under a common reordering of K and V, and reordering
    the queries only moves the output rows: with tau = 1 every block is kept, so
    the clustered path must give dense attention in token order (pins the
    gathers and the scatter back)."""
    r = _rng(30 + iters)
    N, d = 320, 8
    Q = r.standard_normal((1, 2, N, d)) + np.sin(np.arange(N) / 7.0)[None, None, :, None]
    K, V = r.standard_normal((1, 2, N, d)), r.standard_normal((1, 2, N, d))
    O, info = orc.clustered_attention(Q, K, V, 1.0, None, iters)
    assert not np.array_equal(info["perm_q"][0, 0], np.arange(N))      # the order did change
    np.testing.assert_allclose(O, _sdpa64(Q, K, V, False, 1.0 / math.sqrt(d)), rtol=1e-11, atol=1e-12)


def test_clustered_attention_uses_each_side_under_the_others_metric():
    """The set-up of test_kmeans_metric_comes_from_the_other_side on each side in
    turn. Side A: token 0 = (0, 10), tokens 1..63 = 0, tokens 64..127 = (0.9, 10);
    side B: every token (1, 0). Clustered under side B's metric, side A keeps
    the identity order (token 0 stays with block 0); under its own metric token 0
    would move to the second cluster. Side B's tokens are all equal, so its order
    is the identity too (ties go to the first cluster). Checked with A as the
    queries and with A as the keys."""
    A = np.zeros((1, 1, 128, 2))
    A[0, 0, 0] = [0.0, 10.0]
    A[0, 0, 64:] = [0.9, 10.0]
    Bside = np.zeros((1, 1, 128, 2)); Bside[..., 0] = 1.0
    V = _rng(2).standard_normal((1, 1, 128, 2))
    ident = np.arange(128)
    _, info = orc.clustered_attention(A, Bside, V, 0.9, None, 1)
    np.testing.assert_array_equal(info["perm_q"][0, 0], ident)
    np.testing.assert_array_equal(info["perm_k"][0, 0], ident)
    _, info = orc.clustered_attention(Bside, A, V, 0.9, None, 1)
    np.testing.assert_array_equal(info["perm_k"][0, 0], ident)
    np.testing.assert_array_equal(info["perm_q"][0, 0], ident)
    moved = orc.cluster_permutation(orc.kmeans_interaction(A, A, 1)[0])[0, 0]
    assert moved[63] == 0                                     # own metric: token 0 leaves block 0


def test_kmeans_heads_are_independent():
    """Each (batch, head) is clustered on its own: a [2, 2] batch gives what the
    four heads give one by one (pins the per-head Gram matrix and indexing)."""
    r = _rng(17)
    X = r.standard_normal((2, 2, 150, 6)) + np.linspace(0, 2, 150)[None, None, :, None]
    Y = r.standard_normal((2, 2, 150, 6)) * np.array([0.5, 1.0, 1.5, 2.0]).reshape(2, 2, 1, 1)
    a, c, _ = orc.kmeans_interaction(X, Y, 2)
    for b in range(2):
        for h in range(2):
            a1, c1, _ = orc.kmeans_interaction(X[b:b + 1, h:h + 1], Y[b:b + 1, h:h + 1], 2)
            np.testing.assert_array_equal(a[b, h], a1[0, 0])
            np.testing.assert_allclose(c[b, h], c1[0, 0], rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------- replay of recorded decisions
def _brute_force_replay(Q, K, V, mask, decide, causal):
    """Reference-free output of the tiled loop under given skip decisions: per
    row, block energies against one fixed reference (the row's largest visible
    score); the output is the unskipped blocks' weighted V over the energy of
    every visited block (a skipped block stays in the sum, only P.V is dropped)."""
    B, H, N, d = Q.shape
    scale = 1.0 / math.sqrt(d)
    Nb = orc.n_blocks(N)
    O = np.zeros_like(V)
    for b in range(B):
        for h in range(H):
            for i in range(Nb):
                s, e = i * 64, min(N, i * 64 + 64)
                S = scale * Q[b, h, s:e] @ K[b, h].T
                vis = np.repeat(mask[b, h, i].astype(bool), 64)[:N][None, :].repeat(e - s, 0)
                if causal:
                    vis &= np.arange(N)[None, :] <= np.arange(s, e)[:, None]
                S = np.where(vis, S, -np.inf)
                M = S.max(axis=1)
                W = np.exp(S - M[:, None])
                num = np.zeros((e - s, V.shape[-1]))
                for j in np.nonzero(mask[b, h, i])[0]:
                    cols = slice(j * 64, min(N, j * 64 + 64))
                    if not vis[:, cols].any() or decide[b, h, i, j]:
                        continue
                    num += W[:, cols] @ V[b, h, cols]
                O[b, h, s:e] = num / W.sum(axis=1)[:, None]
    return O


@pytest.mark.parametrize("causal", [False, True])
def test_forced_decisions_replay_brute_force(causal):
    """Any decision map, replayed by either filter's loop, gives the brute-force
    output for those decisions (the filter's own test plays no part); replaying
    the loop's own decisions reproduces its unforced output exactly; and each
    reported own decision agrees with the sign of its margin."""
    N, d = 449, 16
    Q, K, V, mask = _recall_case(N + int(causal), N, d, causal, 2)
    Nb = orc.n_blocks(N)
    r = _rng(23)
    forced = (r.random(mask.shape) < 0.4).astype(np.uint8)
    want = _brute_force_replay(Q, K, V, mask, forced, causal)
    got_l = orc.attention_tiled(Q, K, V, mask, -3.0, None, causal, forced=forced)
    got_r = orc.attention_recall(Q, K, V, mask, 0.9, None, causal, forced=forced)
    np.testing.assert_allclose(got_l, want, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(got_r, want, rtol=1e-10, atol=1e-12)
    for fn, arg, strict in ((orc.attention_tiled, -3.0, True), (orc.attention_recall, 0.9, False)):
        O, st = fn(Q, K, V, mask, arg, None, causal, return_stats=True)
        own = np.zeros(mask.shape, dtype=np.uint8)
        for b, h, i, j, sk, mg in st["decisions"]:
            own[b, h, i, j] = sk
            assert sk == ((mg > 0) if strict else (mg >= 0))
        assert own.sum() == st["pv_skipped"] > 0
        np.testing.assert_array_equal(fn(Q, K, V, mask, arg, None, causal, forced=own), O)
        np.testing.assert_allclose(O, _brute_force_replay(Q, K, V, mask, own, causal), rtol=1e-10, atol=1e-12)
    assert Nb > 4


# ---------------------------------------------------------------- INT8 quantization
def test_quantize_blocks_int8_hand_values_and_ties():
    """One block whose amax is 127 (scale exactly 1): the codes are x rounded to
    the nearest integer with ties to even (0.5 -> 0, 1.5 -> 2, 2.5 -> 2, -3.5 -> -4),
    and the amax element maps to +-127 exactly; an all-zero block gets scale 1 and
    codes 0; a second block scaled by 2^-3 gets the same codes and scale 2^-3."""
    row = np.array([127.0, 0.5, 1.5, 2.5, -3.5, -127.0, 0.49, 126.6])
    X = np.zeros((1, 1, 192, 8))
    X[0, 0, 0] = row
    X[0, 0, 64] = row * 0.125
    codes, scales = orc.quantize_blocks_int8(X)
    np.testing.assert_array_equal(codes[0, 0, 0], [127, 0, 2, 2, -4, -127, 0, 127])
    np.testing.assert_array_equal(codes[0, 0, 64], codes[0, 0, 0])
    np.testing.assert_array_equal(scales[0, 0], [1.0, 0.125, 1.0])
    assert np.all(codes[0, 0, 128:] == 0)


def test_quantize_blocks_int8_error_bound_and_range():
    """Random blocks: every code is an integer in [-127, 127], the block's amax
    element reaches +-127, and the dequantized value is within half a step
    (scale / 2, plus fp32 rounding) of x."""
    r = _rng(31)
    X = r.standard_normal((2, 3, 300, 16)) * np.exp(r.uniform(-4, 4, (2, 3, 300, 1)))
    X = X.astype(np.float32).astype(np.float64)
    codes, scales = orc.quantize_blocks_int8(X)
    assert np.array_equal(codes, np.round(codes)) and np.abs(codes).max() <= 127
    nb = orc.n_blocks(300)
    for b in range(2):
        for h in range(3):
            for i in range(nb):
                sl = slice(i * 64, min(300, i * 64 + 64))
                c, x, sc = codes[b, h, sl], X[b, h, sl], scales[b, h, i]
                assert np.abs(c).max() == 127
                assert np.abs(c * sc - x).max() <= 0.5 * sc * (1 + 1e-5) + 1e-12


def test_fwd_int8qk_is_fwd_when_q_and_k_are_representable():
    """Inputs that are integers in [-127, 127] times a power of two, each block
    holding a 127: quantization is exact, so fwd_int8qk equals fwd (with and
    without lambda); on generic inputs the two differ."""
    r = _rng(37)
    Q = np.round(r.uniform(-127, 127, (1, 2, 192, 8))) * 2.0 ** -6
    K = np.round(r.uniform(-127, 127, (1, 2, 192, 8))) * 2.0 ** -5
    Q[:, :, ::64, 0] = 127 * 2.0 ** -6
    K[:, :, ::64, 0] = 127 * 2.0 ** -5
    V = r.standard_normal((1, 2, 192, 8))
    mask = np.ones((1, 2, 3, 3), dtype=np.uint8)
    for lam in (None, -2.0):
        np.testing.assert_array_equal(orc.fwd_int8qk(Q, K, V, mask, lam), orc.fwd(Q, K, V, mask, lam))
    Qg, Kg = r.standard_normal((1, 2, 192, 8)), r.standard_normal((1, 2, 192, 8))
    a, b = orc.fwd_int8qk(Qg, Kg, V, mask), orc.fwd(Qg, Kg, V, mask)
    assert 0 < np.abs(a - b).max() < 0.1
