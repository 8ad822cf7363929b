"""Shared checks for the parity tests (comparison logic only; no method arithmetic
beyond reading the oracle's outputs)."""
from __future__ import annotations

import numpy as np
import torch

BAND = 1e-4          # a block whose cumulative energy lies this close to tau may flip
TIE_REL = 1e-6       # near-equal pooled probabilities may swap at the cut-off
MAX_ABS = 2e-2       # output tolerance (bf16 in, fp32 accumulate)
REL_FRO = 1e-2


def to_np(t: torch.Tensor) -> np.ndarray:
    t = t.detach().to("cpu")
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.numpy()


def check_plan_consistency(mask: np.ndarray, count: np.ndarray, idx: np.ndarray | None):
    """count = popcount of the mask row, idx = its ascending nonzero positions (exact)."""
    assert mask.dtype == np.uint8
    assert set(np.unique(mask)).issubset({0, 1})
    np.testing.assert_array_equal(mask.sum(-1).astype(np.int64), count.astype(np.int64))
    if idx is not None:
        Nb = mask.shape[-1]
        flat_m = mask.reshape(-1, Nb)
        flat_i = idx.reshape(-1, Nb)
        flat_c = count.reshape(-1)
        for r in range(flat_m.shape[0]):
            c = int(flat_c[r])
            np.testing.assert_array_equal(flat_i[r, :c], np.nonzero(flat_m[r])[0])


def compare_masks(gpu_mask: np.ndarray, oplan: dict, tau: float):
    """GPU mask vs the oracle's, exact except blocks decided within BAND of tau.

    Returns (rows_differing, excused_blocks). Fails on any unexcused difference or
    a kept set whose oracle energy misses tau by more than BAND."""
    omask = oplan["mask"]
    P = oplan["P"]
    cb, ca = oplan["c_before"], oplan["c_after"]
    Nb = omask.shape[-1]
    diff = gpu_mask != omask
    rows = np.nonzero(diff.reshape(-1, Nb).any(-1))[0]
    gm = gpu_mask.reshape(-1, Nb).astype(bool)
    om = omask.reshape(-1, Nb).astype(bool)
    Pf = P.reshape(-1, Nb)
    cbf, caf = cb.reshape(-1, Nb), ca.reshape(-1, Nb)
    excused = 0
    for r in rows:
        sym = np.nonzero(gm[r] != om[r])[0]
        kept_o = np.nonzero(om[r])[0]
        cutoff_p = Pf[r, kept_o].min() if kept_o.size else 0.0
        for j in sym:
            near_tau = abs(cbf[r, j] - tau) <= BAND or abs(caf[r, j] - tau) <= BAND
            near_tie = abs(Pf[r, j] - cutoff_p) <= TIE_REL * max(cutoff_p, 1e-300)
            assert near_tau or near_tie, (
                f"row {r}: block {j} differs (gpu={gm[r, j]}, oracle={om[r, j]}, "
                f"c_before={cbf[r, j]:.8f}, c_after={caf[r, j]:.8f}, tau={tau})")
            excused += 1
        energy = Pf[r, gm[r]].sum() / Pf[r].sum()
        assert energy >= tau - BAND, f"row {r}: kept energy {energy} < tau {tau}"
    return len(rows), excused


def output_errors(gpu_o: np.ndarray, ref_o: np.ndarray):
    m = np.isfinite(ref_o)
    g, r = gpu_o[m], ref_o[m]
    max_abs = float(np.abs(g - r).max()) if g.size else 0.0
    den = float(np.linalg.norm(r))
    rel = float(np.linalg.norm(g - r) / den) if den > 0 else float(np.linalg.norm(g - r))
    return max_abs, rel


def assert_output_close(gpu_o: np.ndarray, ref_o: np.ndarray, what: str = ""):
    max_abs, rel = output_errors(gpu_o, ref_o)
    assert max_abs <= MAX_ABS and rel <= REL_FRO, f"{what}: max_abs={max_abs:.3e} rel_fro={rel:.3e}"
    return max_abs, rel


LAM_BORDER = 1e-3     # |lam - (rowmax - m)| below this (natural-log units): fp32 may flip the lambda test
RECALL_BORDER = 1e-4  # |((1 - recall) l - sk alpha - e) / l| below this: fp32 may flip the recall test


def check_filter_replay(q, k, v, mask, gpu_out, gpu_dec, *, lam=None, recall=None, causal=False,
                        qblocks=None, what=""):
    """The GPU's P.V filter decisions replayed by the oracle's tiled loop.

    gpu_dec: the kernel's decision map (uint8 [B, H, Nb, Nb], zero-filled before
    the call). The oracle runs the same loop with those decisions forced, so its
    output must match the GPU's at the output tolerance on every computed row;
    and at every visited pair its own test must agree with the GPU's decision
    unless the test's margin is within the fp32 border of zero. Returns
    (oracle stats, flipped decisions)."""
    from oracle import sparse_attn_oracle as orc
    dec = np.asarray(gpu_dec).astype(np.uint8)
    assert not np.any(dec & (np.asarray(mask) == 0)), "decision recorded for a pair that is not kept"
    if recall is not None:
        ref, st = orc.attention_recall(q, k, v, mask, recall, None, causal, qblocks=qblocks, return_stats=True,
                                       forced=dec)
        border = RECALL_BORDER
    else:
        ref, st = orc.attention_tiled(q, k, v, mask, lam, None, causal, qblocks=qblocks, return_stats=True,
                                      forced=dec)
        border = LAM_BORDER
    assert_output_close(to_np(gpu_out) if isinstance(gpu_out, torch.Tensor) else gpu_out, ref, what)
    flips = 0
    for b, h, i, j, own, margin in st["decisions"]:
        if bool(dec[b, h, i, j]) != own:
            assert abs(margin) < border, f"{what}: pair {(b, h, i, j)} decided {dec[b, h, i, j]}, margin {margin}"
            flips += 1
    return st, flips
