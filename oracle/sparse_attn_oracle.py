"""CPU oracle for block-sparse attention with a cumulative-energy block mask.

TEST INFRASTRUCTURE ONLY. This file is the plain, slow, fp64 statement of what the
GPU path computes. Only the tests, the package's smoke check and the benchmark's
CPU-baseline / reference arm may import it; the product path never does. It
shares no code with the CUDA library (it does not import the package).

What it follows:
  * SpargeAttn abstract (page "taxoreview ... dblp:344/2858", repeated in the HF
    Daily Papers listing): a two-stage online filter. Stage 1 predicts the
    attention map cheaply and skips the matmuls of unimportant regions; stage 2 is
    an online-softmax-aware filter that skips further matmuls at no extra cost.
  * "Training-free sparse attention based on cumulative energy filtering"
    (DynSparse news article, method paragraph): keep tokens until a fixed recall of
    the attention energy is reached, with a per-row ("dynamic") threshold derived
    from the cumulative energy instead of a fixed top-k budget or static cut.

Readings where the pages are silent (each is also listed in the design notes):
  * stage 1 pools Q and K by the mean over blocks of 64 tokens; a ragged last block
    is averaged over its valid tokens only;
  * pooled logits use the same softmax scale as the attention;
  * causal: only key blocks j <= i enter the pooled softmax of query block i;
  * selection: sort the row of pooled probabilities in descending order (ties:
    lower block index first), keep the shortest prefix whose running sum reaches
    tau times the row total;
  * stage 2: inside the tiled online-softmax loop (64-row query blocks, kept key
    blocks visited in ascending order), the P.V product of a key block is skipped
    when every valid row r of the query block has rowmax_r(S_blk) - m_r < lam,
    with m_r the running max before the block; the block still enters the
    running max and the running sum l (only P.V is skipped).
  * a query row that ends with no visible key gets an output of zero.
  * in-operator cumulative-energy filter (the DynSparse step placed inside the
    FlashAttention operator; an alternative to the lambda test): the same tiled
    loop, but a key block's P.V is skipped when, for every row of the query block
    that sees it, the energy skipped so far plus the block's own energy stays
    within (1 - recall) of the running sum l including the block; l is the
    cumulative energy the operator already keeps, the threshold moves with it.

Arithmetic is fp64 throughout; inputs are the exact values of the bf16 tensors.

Quantized QK^T (SpargeAttn is "sparse and quantized"; the pages give no scheme,
so this is a design, stated here and pinned by the tests): Q and K are quantized
per (batch, head, 64-token block) to FP8 E4M3 with one scale per block,
s = max|x| / 448 (448 = largest finite E4M3 value), codes = nearest E4M3 value
of x * (448 / max|x|) computed in fp32 (the kernel's precision for this integer
decision), ties to even, saturating. The scores are then the dequantized
(code * s) products; V, P and the rest of the attention are unchanged.

Clustered variant (iCATS abstract: clustering of query and key tokens "based on
query-key dot-product interactions", reformulated "as a simple quadratic form";
the abstract gives no formula, so this is a reading, pinned by the tests):
  * replacing a query q by a centroid c changes its dot products with every key
    k by (q - c).k, and the sum of their squares over the keys is the quadratic
    form (q - c)^T G_K (q - c) with G_K = sum_k k k^T, the keys' Gram matrix; the
    queries are clustered by k-means under that distance, the keys likewise
    under G_Q = sum_q q q^T;
  * ceil(N/64) clusters per side, initialised to the 64-token block means (so
    zero iterations is the plain block pooling); Lloyd iterations assign each
    token to the nearest centroid (ties: lowest cluster index) and move each
    centroid to the mean of its tokens (a cluster left empty keeps its centroid);
  * tokens are then reordered by cluster (stable: ascending token index within a
    cluster) and the clusters packed back to back, so the tail of one cluster
    shares a 64-token block with the head of the next instead of being padded
    ("tail merging"); the plan and the forward run on the reordered Q, K, V and
    the output rows are put back in token order. Non-causal only.

Entry points: block_mean_pool, pooled_logits, pooled_softmax,
cumulative_energy_select, plan, attention_masked, attention_tiled,
attention_recall, fwd, round_e4m3, quantize_blocks_e4m3, fwd_fp8qk, gram, interaction_distance,
kmeans_interaction, cluster_permutation, clustered_attention.
"""
from __future__ import annotations

import math
from typing import Iterable, Optional

import numpy as np

BLOCK = 64


def as_f64(x) -> np.ndarray:
    """Exact fp64 copy of a (possibly bf16 torch) array."""
    if hasattr(x, "detach"):  # torch tensor, any dtype; bf16 -> fp32 -> fp64 is exact
        x = x.detach().to("cpu")
        if str(x.dtype) == "torch.bfloat16":
            x = x.float()
        x = x.numpy()
    return np.asarray(x, dtype=np.float64)


def n_blocks(N: int, block: int = BLOCK) -> int:
    return -(-N // block)


# ---------------------------------------------------------------- stage 1

def block_mean_pool(X: np.ndarray, block: int = BLOCK) -> np.ndarray:
    """Mean of each block of `block` consecutive tokens: [..., N, d] -> [..., Nb, d].

    Stage 1 of the SpargeAttn abstract ("rapidly ... predict the attention map");
    the pooling operator is the mean (reading). A ragged tail block divides by its
    own token count."""
    N = X.shape[-2]
    Nb = n_blocks(N, block)
    out = np.empty(X.shape[:-2] + (Nb, X.shape[-1]), dtype=np.float64)
    for i in range(Nb):
        s, e = i * block, min(N, (i + 1) * block)
        out[..., i, :] = X[..., s:e, :].sum(axis=-2) / (e - s)
    return out


def pooled_logits(Qp: np.ndarray, Kp: np.ndarray, scale: float, causal: bool) -> np.ndarray:
    """L[i, j] = scale * <Qp_i, Kp_j>; with causal, key blocks after the query block
    are excluded (-inf)."""
    L = scale * np.matmul(Qp, np.swapaxes(Kp, -1, -2))
    if causal:
        Nb = L.shape[-1]
        later = np.triu(np.ones((Nb, Nb), dtype=bool), k=1)
        L = np.where(later, -np.inf, L)
    return L


def pooled_softmax(L: np.ndarray) -> np.ndarray:
    """Row softmax of the pooled logits: the predicted block attention map."""
    m = L.max(axis=-1, keepdims=True)
    e = np.exp(L - m)
    return e / e.sum(axis=-1, keepdims=True)


def cumulative_energy_select(P: np.ndarray, tau):
    """Per row of the predicted map, keep the fewest blocks whose energy reaches tau.

    tau is a scalar, or one value per (batch, head) (an array broadcastable to
    P.shape[:-2], e.g. [B, H] or [H]): every row of a head uses its head's tau,
    the per-head recall threshold of an SNR-guided schedule (iCATS abstract).

    DynSparse (cumulative energy filtering): a fixed recall of the attention energy
    is kept, and the per-row cut-off value (the smallest kept probability) is the
    dynamic threshold. Steps: sort descending with ties to the lower index (stable
    sort of -p), running sum c_r, first r with c_r >= tau * c_last, keep that prefix.

    Returns mask (uint8, [..., Nb, Nb]), count (int64 [..., Nb]), idx (int64,
    ascending kept indices, padded with -1) and, per block in its original
    position, the row's running sum just before (`c_before`) and after (`c_after`)
    that block in sorted order, normalised by the row total; these mark the blocks
    whose fate is decided within rounding of tau.
    """
    shape = P.shape
    rows = P.reshape(-1, shape[-1])
    Nb = shape[-1]
    mask = np.zeros(rows.shape, dtype=np.uint8)
    count = np.zeros(rows.shape[0], dtype=np.int64)
    idx = np.full(rows.shape, -1, dtype=np.int64)
    c_before = np.zeros(rows.shape, dtype=np.float64)
    c_after = np.zeros(rows.shape, dtype=np.float64)
    tau_rows = np.broadcast_to(np.asarray(tau, dtype=np.float64)[..., None], shape[:-1]).reshape(-1)
    for r in range(rows.shape[0]):
        p = rows[r]
        order = np.argsort(-p, kind="stable")
        c = np.cumsum(p[order])
        total = c[-1]
        hit = np.nonzero(c >= tau_rows[r] * total)[0]
        rstar = int(hit[0]) + 1 if hit.size else Nb
        kept = np.sort(order[:rstar])
        mask[r, kept] = 1
        count[r] = rstar
        idx[r, :rstar] = kept
        c_after[r, order] = c / total
        c_before[r, order] = (c - p[order]) / total
    return (mask.reshape(shape), count.reshape(shape[:-1]), idx.reshape(shape),
            c_before.reshape(shape), c_after.reshape(shape))


def plan(Q, K, tau, scale: Optional[float] = None, causal: bool = False,
         block: int = BLOCK) -> dict:
    """Stage 1 end to end: pool, pooled logits, pooled softmax, cumulative-energy
    selection. Q, K: [B, H, N, d]; tau a scalar or one value per (batch, head)."""
    Q = as_f64(Q)
    K = as_f64(K)
    d = Q.shape[-1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    Qp = block_mean_pool(Q, block)
    Kp = block_mean_pool(K, block)
    L = pooled_logits(Qp, Kp, scale, causal)
    P = pooled_softmax(L)
    mask, count, idx, cb, ca = cumulative_energy_select(P, tau)
    return dict(Qp=Qp, Kp=Kp, L=L, P=P, mask=mask, count=count, idx=idx,
                c_before=cb, c_after=ca)


# ---------------------------------------------------------------- stage 2

def _visible(mask_row: np.ndarray, N: int, block: int) -> np.ndarray:
    """Token-level key visibility of one query block from its block-mask row."""
    vis = np.repeat(mask_row.astype(bool), block)[:N]
    return vis


def attention_masked(Q, K, V, mask, scale: Optional[float] = None, causal: bool = False,
                     block: int = BLOCK, qblocks: Optional[Iterable[int]] = None):
    """Stage-2 output without the lambda filter: for each query token t, softmax
    attention over the keys of the blocks its query block keeps (and s <= t when
    causal). Returns O [B, H, N, d] (rows of query blocks not in `qblocks` are NaN)."""
    Q, K, V = as_f64(Q), as_f64(K), as_f64(V)
    mask = np.asarray(mask)
    B, H, N, d = Q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    Nb = n_blocks(N, block)
    qbs = range(Nb) if qblocks is None else qblocks
    O = np.full((B, H, N, V.shape[-1]), np.nan)
    for b in range(B):
        for h in range(H):
            for i in qbs:
                s, e = i * block, min(N, (i + 1) * block)
                vis = _visible(mask[b, h, i], N, block)
                S = scale * Q[b, h, s:e] @ K[b, h].T           # [rows, N]
                allow = np.broadcast_to(vis, S.shape).copy()
                if causal:
                    allow &= np.arange(N)[None, :] <= np.arange(s, e)[:, None]
                S = np.where(allow, S, -np.inf)
                m = S.max(axis=1, keepdims=True)
                none = ~np.isfinite(m[:, 0])
                m[none] = 0.0
                W = np.exp(S - m)
                lsum = W.sum(axis=1, keepdims=True)
                out = (W @ V[b, h]) / np.where(lsum > 0, lsum, 1.0)
                out[none] = 0.0
                O[b, h, s:e] = out
    return O


def attention_tiled(Q, K, V, mask, lam: float, scale: Optional[float] = None,
                    causal: bool = False, block: int = BLOCK,
                    qblocks: Optional[Iterable[int]] = None, return_stats: bool = False,
                    forced=None):
    """Stage 2 with the online-softmax-aware filter, as a literal fp64 run of the
    tiled loop: per 64-row query block, kept key blocks in ascending order,
    running max m, running sum l, accumulator O.

    SpargeAttn abstract, second stage: a block whose P.V contribution is
    negligible under the current running max is skipped at no extra cost. The
    test is rowmax_r(S_blk) - m_r < lam for every row r of the query block that
    sees at least one key of the block (m_r before the block, natural-log units
    of the scaled logits); only P.V is skipped, m and l are still updated.
    lam = -inf never skips, and then this equals attention_masked.

    forced [B, H, Nb, Nb] (0/1), if given, replaces the test: the pair (i, j) is
    skipped iff forced[b, h, i, j] is nonzero (a replay of decisions recorded
    elsewhere; the test is still evaluated and reported). The filter's reading
    allows a decision taken in lower precision to flip only where the test's
    margin is within rounding of zero, which the caller checks on the margins.

    With return_stats, also returns dict(kept_pairs, pv_skipped, decisions): a
    list of (b, h, i, j, own_skip, margin) with margin = lam - max over the
    seeing rows of (rowmax - m) (the test says "skip" iff margin > 0; +inf for a
    row's first block, which is never skipped, is reported as -inf)."""
    Q, K, V = as_f64(Q), as_f64(K), as_f64(V)
    mask = np.asarray(mask)
    B, H, N, d = Q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    Nb = n_blocks(N, block)
    qbs = range(Nb) if qblocks is None else qblocks
    O = np.full((B, H, N, V.shape[-1]), np.nan)
    kept_pairs = 0
    skipped_pairs = 0
    decisions = []
    for b in range(B):
        for h in range(H):
            for i in qbs:
                s, e = i * block, min(N, (i + 1) * block)
                rows = np.arange(s, e)
                m = np.full(e - s, -np.inf)
                l = np.zeros(e - s)
                acc = np.zeros((e - s, V.shape[-1]))
                for j in np.nonzero(mask[b, h, i])[0]:
                    ks, ke = j * block, min(N, (j + 1) * block)
                    S = scale * Q[b, h, s:e] @ K[b, h, ks:ke].T
                    if causal:
                        S = np.where(np.arange(ks, ke)[None, :] <= rows[:, None], S, -np.inf)
                    rmax = S.max(axis=1)
                    sees = np.isfinite(rmax)
                    if not sees.any():
                        continue
                    kept_pairs += 1
                    with np.errstate(invalid="ignore"):
                        diff = rmax - m                      # +inf where m = -inf
                    own = bool(np.all(diff[sees] < lam))
                    decisions.append((b, h, i, int(j), own, float(lam - diff[sees].max())))
                    skip = own if forced is None else bool(forced[b, h, i, j])
                    m_new = np.maximum(m, rmax)
                    ref = np.where(np.isfinite(m_new), m_new, 0.0)
                    alpha = np.where(np.isfinite(m), np.exp(m - ref), 0.0)
                    Pb = np.exp(S - ref[:, None])
                    l = l * alpha + Pb.sum(axis=1)
                    acc = acc * alpha[:, None]
                    if skip:
                        skipped_pairs += 1
                    else:
                        acc = acc + Pb @ V[b, h, ks:ke]
                    m = m_new
                out = acc / np.where(l > 0, l, 1.0)[:, None]
                out[l <= 0] = 0.0
                O[b, h, s:e] = out
    if return_stats:
        return O, dict(kept_pairs=kept_pairs, pv_skipped=skipped_pairs, decisions=decisions)
    return O


def attention_recall(Q, K, V, mask, recall: float, scale: Optional[float] = None,
                     causal: bool = False, block: int = BLOCK,
                     qblocks: Optional[Iterable[int]] = None, return_stats: bool = False,
                     forced=None):
    """Stage 2 with the in-operator cumulative-energy filter, as a literal fp64 run
    of the tiled loop (64-row query blocks, kept key blocks in ascending order).

    DynSparse article: a fixed recall of the attention energy is enough for
    accuracy, and the threshold is a dynamic one derived from the cumulative
    energy of the selected tokens, which the FlashAttention operator already holds
    (its running sum l). Reading: per row r, l_r is the energy seen so far and
    sk_r the part of it whose P.V was skipped, both relative to the running max.
    For key block j with row energies e_r = sum_c exp(S_rc - m'_r), the block's
    P.V is skipped when every row r of the query block that sees a key of the
    block has sk_r * alpha_r + e_r <= (1 - recall) * (l_r * alpha_r + e_r)
    (alpha_r = exp(m_r - m'_r) rescales the old sums to the new max). l always
    takes e_r; sk takes it only when the block is skipped. By induction
    sk_r <= (1 - recall) * l_r after every block, so each row keeps at least the
    fraction `recall` of the energy of the blocks it visits.

    With return_stats, also returns dict(kept_pairs, pv_skipped, decisions,
    recall_rows): decisions is a list of (b, h, i, j, skipped, margin) where
    margin = min over the seeing rows of ((1 - recall) * l' - (sk * alpha + e)) / l'
    (the decision is "skip" iff margin >= 0), and recall_rows [B, H, N] is
    1 - sk / l per row at the end (NaN for rows not computed).

    forced [B, H, Nb, Nb] (0/1), if given, replaces the test as in
    attention_tiled: pair (i, j) is skipped iff forced[b, h, i, j] is nonzero, and
    sk, l and the output follow that decision; `decisions` still reports the
    test's own verdict and margin for each pair."""
    Q, K, V = as_f64(Q), as_f64(K), as_f64(V)
    mask = np.asarray(mask)
    B, H, N, d = Q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    Nb = n_blocks(N, block)
    qbs = range(Nb) if qblocks is None else qblocks
    O = np.full((B, H, N, V.shape[-1]), np.nan)
    rec_rows = np.full((B, H, N), np.nan)
    kept_pairs = 0
    skipped_pairs = 0
    decisions = []
    budget = 1.0 - recall
    for b in range(B):
        for h in range(H):
            for i in qbs:
                s, e = i * block, min(N, (i + 1) * block)
                rows = np.arange(s, e)
                m = np.full(e - s, -np.inf)
                l = np.zeros(e - s)
                sk = np.zeros(e - s)
                acc = np.zeros((e - s, V.shape[-1]))
                for j in np.nonzero(mask[b, h, i])[0]:
                    ks, ke = j * block, min(N, (j + 1) * block)
                    S = scale * Q[b, h, s:e] @ K[b, h, ks:ke].T
                    if causal:
                        S = np.where(np.arange(ks, ke)[None, :] <= rows[:, None], S, -np.inf)
                    rmax = S.max(axis=1)
                    sees = np.isfinite(rmax)
                    if not sees.any():
                        continue
                    kept_pairs += 1
                    m_new = np.maximum(m, rmax)
                    ref = np.where(np.isfinite(m_new), m_new, 0.0)
                    alpha = np.where(np.isfinite(m), np.exp(m - ref), 0.0)
                    Pb = np.exp(S - ref[:, None])
                    en = Pb.sum(axis=1)
                    l_new = l * alpha + en
                    sk_try = sk * alpha + en
                    room = budget * l_new - sk_try
                    margin = float(np.min(room[sees] / l_new[sees]))
                    own = bool(np.all(room[sees] >= 0.0))
                    decisions.append((b, h, i, int(j), own, margin))
                    skip = own if forced is None else bool(forced[b, h, i, j])
                    l = l_new
                    acc = acc * alpha[:, None]
                    if skip:
                        skipped_pairs += 1
                        sk = sk_try
                    else:
                        sk = sk * alpha
                        acc = acc + Pb @ V[b, h, ks:ke]
                    m = m_new
                out = acc / np.where(l > 0, l, 1.0)[:, None]
                out[l <= 0] = 0.0
                O[b, h, s:e] = out
                with np.errstate(invalid="ignore", divide="ignore"):
                    rec_rows[b, h, s:e] = np.where(l > 0, 1.0 - sk / np.where(l > 0, l, 1.0), 1.0)
    if return_stats:
        return O, dict(kept_pairs=kept_pairs, pv_skipped=skipped_pairs, decisions=decisions,
                       recall_rows=rec_rows)
    return O


def fwd(Q, K, V, mask, lam: Optional[float] = None, scale: Optional[float] = None,
        causal: bool = False, block: int = BLOCK, qblocks=None, forced=None):
    """Stage 2: the masked attention, with the lambda filter when lam is finite
    (forced: a replay of recorded filter decisions, see attention_tiled)."""
    if lam is None or lam == -math.inf:
        return attention_masked(Q, K, V, mask, scale, causal, block, qblocks)
    return attention_tiled(Q, K, V, mask, lam, scale, causal, block, qblocks, forced=forced)


# ----------------------------------------------------------------------------
# FP8 E4M3 quantization of Q and K (see the module docstring)
E4M3_MAX = 448.0


def round_e4m3(x) -> np.ndarray:
    """Nearest FP8 E4M3 value of x (fp64 result), ties to even, saturating at
    +-448. E4M3: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits, no
    infinities. In the binade [2^e, 2^(e+1)) (e >= -6) the representable values are
    spaced 2^(e-3); below 2^-6 the subnormals are spaced 2^-9 as well."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    _, ex = np.frexp(np.maximum(a, 2.0 ** -6))      # a = m * 2^ex with m in [0.5, 1)
    step = np.ldexp(1.0, ex - 1 - 3)
    r = np.minimum(np.round(a / step) * step, E4M3_MAX)   # np.round: half to even
    return np.copysign(r, x)


def quantize_blocks_e4m3(X, block: int = BLOCK):
    """Per (batch, head, block of 64 tokens) E4M3 quantization of X [B, H, N, d]:
    amax = max |x| over the block, scale = amax / 448 and codes =
    round_e4m3(x * (448 / amax)), both in fp32 (scale 1 and codes 0 for an
    all-zero block). Returns (codes as fp64 values [B, H, N, d], scales fp64
    [B, H, Nb]); code * scale is the dequantized value."""
    X32 = np.asarray(as_f64(X), dtype=np.float32)
    B, H, N, d = X32.shape
    nb = n_blocks(N, block)
    codes = np.zeros((B, H, N, d))
    scales = np.ones((B, H, nb))
    for i in range(nb):
        sl = slice(i * block, min(N, (i + 1) * block))
        amax = np.abs(X32[:, :, sl, :]).max(axis=(2, 3))
        pos = amax > 0
        inv = np.where(pos, np.float32(E4M3_MAX) / np.where(pos, amax, np.float32(1)), np.float32(0))
        inv = inv.astype(np.float32)
        y = (X32[:, :, sl, :] * inv[:, :, None, None]).astype(np.float32)
        codes[:, :, sl, :] = round_e4m3(y)
        scales[:, :, i] = np.where(pos, (amax / np.float32(E4M3_MAX)).astype(np.float32), 1.0)
    return codes, scales


# ----------------------------------------------------------------------------
# INT8 quantization of Q and K (symmetric, one scale per 64-token block)
INT8_MAX = 127.0


def quantize_blocks_int8(X, block: int = BLOCK):
    """Per (batch, head, block of 64 tokens) symmetric INT8 quantization of X
    [B, H, N, d]: amax = max |x| over the block, scale = amax / 127, and codes =
    x * (127 / amax) rounded to the nearest integer (ties to even); the product
    and the scale are formed in fp32 (scale 1 and codes 0 for an all-zero
    block). |code| <= 127, so -128 never occurs. Returns (codes as fp64 values
    [B, H, N, d], scales fp64 [B, H, Nb]); code * scale is the dequantized value."""
    X32 = np.asarray(as_f64(X), dtype=np.float32)
    B, H, N, d = X32.shape
    nb = n_blocks(N, block)
    codes = np.zeros((B, H, N, d))
    scales = np.ones((B, H, nb))
    for i in range(nb):
        sl = slice(i * block, min(N, (i + 1) * block))
        amax = np.abs(X32[:, :, sl, :]).max(axis=(2, 3))
        pos = amax > 0
        inv = np.where(pos, np.float32(INT8_MAX) / np.where(pos, amax, np.float32(1)), np.float32(0))
        inv = inv.astype(np.float32)
        y = (X32[:, :, sl, :] * inv[:, :, None, None]).astype(np.float32).astype(np.float64)
        codes[:, :, sl, :] = np.clip(np.round(y), -INT8_MAX, INT8_MAX)   # np.round: half to even
        scales[:, :, i] = np.where(pos, (amax / np.float32(INT8_MAX)).astype(np.float32), 1.0)
    return codes, scales


def fwd_int8qk(Q, K, V, mask, lam: Optional[float] = None, scale: Optional[float] = None,
               causal: bool = False, block: int = BLOCK, qblocks=None, forced=None):
    """Stage 2 with INT8 scores: fwd on the dequantized Q and K (codes times their
    block scale), V as given. The mask comes from the unquantized plan."""
    cq, sq = quantize_blocks_int8(Q, block)
    ck, sk = quantize_blocks_int8(K, block)
    N = cq.shape[2]
    tok = np.minimum(np.arange(N) // block, sq.shape[2] - 1)
    Qd = cq * sq[:, :, tok][..., None]
    Kd = ck * sk[:, :, tok][..., None]
    return fwd(Qd, Kd, V, mask, lam, scale, causal, block, qblocks, forced=forced)


def fwd_fp8qk(Q, K, V, mask, lam: Optional[float] = None, scale: Optional[float] = None,
              causal: bool = False, block: int = BLOCK, qblocks=None):
    """Stage 2 with quantized scores: fwd on the dequantized Q and K (codes times
    their block scale), V as given. The mask comes from the unquantized plan."""
    cq, sq = quantize_blocks_e4m3(Q, block)
    ck, sk = quantize_blocks_e4m3(K, block)
    N = cq.shape[2]
    tok = np.minimum(np.arange(N) // block, sq.shape[2] - 1)
    Qd = cq * sq[:, :, tok][..., None]
    Kd = ck * sk[:, :, tok][..., None]
    return fwd(Qd, Kd, V, mask, lam, scale, causal, block, qblocks)



# ----------------------------------------------------------------------------
# Clustering by query-key interaction (see the module docstring)

def gram(Y) -> np.ndarray:
    """Gram matrix sum_t y_t y_t^T of the tokens of Y [..., N, d]: [..., d, d]."""
    Y = as_f64(Y)
    return np.swapaxes(Y, -1, -2) @ Y


def interaction_distance(X, C, G) -> np.ndarray:
    """(x - c)^T G (x - c) for every token x of X [..., N, d] and centroid c of
    C [..., M, d] under G [..., d, d]: [..., N, M]. Expanded as
    x^T G x - 2 x^T G c + c^T G c (the tests check it against the sum over the
    other side's tokens of ((x - c).y)^2)."""
    X, C, G = as_f64(X), as_f64(C), as_f64(G)
    XG = X @ G
    xx = np.sum(XG * X, axis=-1)[..., :, None]
    cc = np.sum((C @ G) * C, axis=-1)[..., None, :]
    return xx - 2.0 * XG @ np.swapaxes(C, -1, -2) + cc


def kmeans_interaction(X, Y, iters: int, block: int = BLOCK):
    """k-means of the tokens of X [B, H, N, d] under the metric G = gram(Y) of the
    other side, per (batch, head): ceil(N/block) clusters, initialised to the
    block means, `iters` Lloyd iterations. Returns (assign int64 [B, H, N],
    centroids [B, H, C, d], objective list of length iters + 1: the sum over the
    tokens of the distance to their centroid, after the initial assignment to
    the blocks and after each iteration)."""
    X, Y = as_f64(X), as_f64(Y)
    B, H, N, d = X.shape
    nc = n_blocks(N, block)
    G = gram(Y)
    cent = block_mean_pool(X, block)
    assign = np.broadcast_to(np.arange(N) // block, (B, H, N)).copy()

    def objective(a, c):
        dist = interaction_distance(X, c, G)
        return float(np.take_along_axis(dist, a[..., None], axis=-1).sum())

    obj = [objective(assign, cent)]
    for _ in range(iters):
        dist = interaction_distance(X, cent, G)
        assign = np.argmin(dist, axis=-1)                  # first minimum: lowest index
        new = cent.copy()
        for b in range(B):
            for h in range(H):
                for c in range(nc):
                    members = assign[b, h] == c
                    if members.any():
                        new[b, h, c] = X[b, h, members].mean(axis=0)
        cent = new
        obj.append(objective(assign, cent))
    return assign, cent, obj


def cluster_permutation(assign) -> np.ndarray:
    """perm[..., p] = the token at position p once the tokens are ordered by
    cluster, ascending token index within a cluster (a stable sort)."""
    return np.argsort(np.asarray(assign), axis=-1, kind="stable")


def clustered_attention(Q, K, V, tau, lam: Optional[float] = None, iters: int = 2,
                        scale: Optional[float] = None, block: int = BLOCK, perms=None):
    """Plan + forward on tokens reordered by interaction clustering, output in
    token order. Queries are clustered under gram(K), keys under gram(Q); K and V
    share the key order. `perms` = (perm_q, perm_k) replaces the clustering (for
    checking an output against a given ordering). Returns (O [B, H, N, d], dict
    with perm_q, perm_k, the plan on the reordered tokens)."""
    Q, K, V = as_f64(Q), as_f64(K), as_f64(V)
    if perms is None:
        aq, _, _ = kmeans_interaction(Q, K, iters, block)
        ak, _, _ = kmeans_interaction(K, Q, iters, block)
        pq, pk = cluster_permutation(aq), cluster_permutation(ak)
    else:
        pq, pk = (np.asarray(p, dtype=np.int64) for p in perms)
    Qs = np.take_along_axis(Q, pq[..., None], axis=2)
    Ks = np.take_along_axis(K, pk[..., None], axis=2)
    Vs = np.take_along_axis(V, pk[..., None], axis=2)
    p = plan(Qs, Ks, tau, scale, False, block)
    Os = fwd(Qs, Ks, Vs, p["mask"], lam, scale, False, block)
    O = np.empty_like(Os)
    np.put_along_axis(O, pq[..., None], Os, axis=2)
    return O, dict(perm_q=pq, perm_k=pk, plan=p)
