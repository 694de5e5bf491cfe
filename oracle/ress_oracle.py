"""CPU oracle for block-sparse global attention: pooled block selection,
block-sparse attention and per-dropped-block drift.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The CUDA library
never calls it and shares no code with it; the two meet only through the
seeded inputs of ``block_sparse_global_mean_b200.workloads``.

Everything is plain numpy in float64, written step by step in the order the
definition gives, with no blocking, fusion or reordering.  A matmul, a sort
and ``exp``/``log`` are the only library primitives used.

Sources (the pages carry no equations; the operations are the ones the pages
name, made exact as stated per function):

* ReSS: Residual-Restoring Sparse Attention for 3D Vision Transformers
  (thelatestinai.com), Abstract, Fig. 1, Fig. 3, Fig. 9, Table 1, Table S5,
  Table S6.
* VASC: Value-Aware Sparse Attention with Cross-Layer Memory
  (paperlayer.ai), sections 4.1, 4.2, A.1, A.2, A.3.

Readings taken where the pages are silent (each is repeated at its function):

* the pooled score is softmax over all nb key blocks of (Qbar . Kbar) / sqrt(d),
  d the head dimension;
* the value contrast is the L2 norm of Vbar_j - Vbar_{j-1} with the global
  predecessor j-1 (crossing view boundaries) and c_0 = 0, added to the
  probability with weight lambda;
* top-k keeps the k largest scores, ties to the lower block index, and lists
  the kept blocks in ascending order;
* attention is bidirectional (no causal mask) and normalised over the kept
  tokens only; lse is the natural-log sum of exp over the kept logits;
* the drift contribution of a dropped block uses the kept-set normaliser lse;
  its norm is the Frobenius norm over the block's B x d contribution matrix, and
  the drop-set drift J is the Frobenius norm of the summed contributions.
* the CDF threshold keeps the fewest top blocks whose probabilities reach tau
  (ties to the lower index; every block if the total never reaches tau);
* with padding and special tokens: blocks pool their valid tokens only,
  padding keys never enter a softmax and padding queries write nothing,
  special (camera, register) queries attend densely to every valid key,
  key blocks made only of special tokens are always kept, and special queries
  drop nothing in the drift.

Every function here is pinned by the tests in ``tests/test_oracle_pins.py``
against closed forms, brute force, invariants or independent library routines.
The numeric tolerances of the drift comparison (not its values) are not fixed
by the pages.
"""

from __future__ import annotations

import math
from typing import Iterable, Optional, Sequence, Tuple

import numpy as np


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------------------
# Stage 1: selection
# ---------------------------------------------------------------------------

def pool_blocks(x, block: int) -> np.ndarray:
    """Mean of each run of ``block`` consecutive tokens, per head.

    ``x`` is ``[N, H, d]``; returns ``[H, nb, d]`` with
    out[h, i] = (1/B) * sum_{t = iB}^{iB+B-1} x[t, h].

    The pooled query/key inner products of SparseVGGT are the selection basis
    (ReSS, Table S5, SpargeAttn row); VASC pools queries, keys and values per
    native block (VASC, sections 4.1 and A.1).
    """
    x = _f64(x)
    n, h, d = x.shape
    assert n % block == 0, "N must be a multiple of the block size"
    nb = n // block
    sums = x.reshape(nb, block, h, d).sum(axis=1)          # [nb, H, d]
    return np.ascontiguousarray((sums / block).transpose(1, 0, 2))


def block_logits(qbar, kbar) -> np.ndarray:
    """Pooled logits s[h, i, j] = (Qbar[h, i] . Kbar[h, j]) / sqrt(d).

    Reading: the temperature is sqrt(d) with d the head dimension, the usual
    attention scale, applied to the pooled vectors.
    """
    qbar = _f64(qbar)
    kbar = _f64(kbar)
    d = qbar.shape[-1]
    return np.matmul(qbar, kbar.transpose(0, 2, 1)) / math.sqrt(d)


def block_probs(logits) -> np.ndarray:
    """Softmax over all nb key blocks of each (head, query block) row."""
    s = _f64(logits)
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / e.sum(axis=-1, keepdims=True)


def value_contrast(vbar) -> np.ndarray:
    """c[h, j] = || Vbar[h, j] - Vbar[h, j-1] ||_2 for j >= 1 and c[h, 0] = 0.

    VASC measures the contrast between neighbouring pooled value blocks
    (VASC, sections 4.1 and A.3).  Reading: the plain L2 norm with the global
    predecessor j-1, and zero contrast for the first block, which has no
    predecessor (VASC A.3 gives an unpaired block zero contrast).
    """
    vbar = _f64(vbar)
    h, nb, _ = vbar.shape
    c = np.zeros((h, nb), dtype=np.float64)
    if nb > 1:
        diff = vbar[:, 1:, :] - vbar[:, :-1, :]
        c[:, 1:] = np.sqrt((diff * diff).sum(axis=-1))
    return c


def selection_scores(q, k, v, block: int, lam: float):
    """The ranked quantity of the selection and its parts.

    Returns a dict with ``logits`` [H, nb, nb], ``probs`` [H, nb, nb],
    ``contrast`` [H, nb] (zeros when lam == 0) and ``score`` [H, nb, nb] =
    probs + lam * contrast[h, None, j].

    Reading: the contrast term is added to the probability (VASC section 4.1
    says the contrast modulates the relevance; the additive form is taken).
    """
    qbar = pool_blocks(q, block)
    kbar = pool_blocks(k, block)
    logits = block_logits(qbar, kbar)
    probs = block_probs(logits)
    if lam != 0.0:
        assert v is not None, "the value contrast needs V"
        contrast = value_contrast(pool_blocks(v, block))
    else:
        contrast = np.zeros(probs.shape[:2], dtype=np.float64)
    score = probs + lam * contrast[:, None, :]
    return {"logits": logits, "probs": probs, "contrast": contrast, "score": score}


def topk_lowest_index(score, budget: int) -> np.ndarray:
    """Indices of the ``budget`` largest entries of each row, ascending.

    A binary Top-K mask with exact capacity (VASC, section A.2): every row keeps
    exactly ``budget`` blocks.  Ties go to the lower block index: a stable sort
    on the negated score keeps equal scores in index order.
    """
    score = _f64(score)
    order = np.argsort(-score, axis=-1, kind="stable")[..., :budget]
    return np.sort(order, axis=-1).astype(np.int32)


def select_blocks(q, k, v, block: int, budget: int, lam: float = 0.0,
                  return_scores: bool = False):
    """Stage 1 end to end: idx [H, nb, budget] int32, ascending per row."""
    sc = selection_scores(q, k, v, block, lam)
    idx = topk_lowest_index(sc["score"], budget)
    if return_scores:
        return idx, sc
    return idx


def cdf_counts(probs, tau: float) -> np.ndarray:
    """Per row, how many blocks the cumulative (CDF) threshold keeps.

    SparseVGGT keeps, for every query block, the key blocks of largest pooled
    probability until their cumulative mass reaches a threshold (ReSS, Table S5:
    with the similarity gate off, selection reduces to a cumulative threshold on
    pooled query/key inner products; Table 2, row "+ CDF threshold").
    Reading: blocks in descending probability, ties to the lower index; the
    count is the smallest m >= 1 whose first m probabilities sum to at least
    tau; every block when the rounded total never reaches tau.
    """
    p = _f64(probs)
    nb = p.shape[-1]
    order = np.argsort(-p, axis=-1, kind="stable")
    cum = np.cumsum(np.take_along_axis(p, order, axis=-1), axis=-1)
    reached = cum >= tau
    first = np.argmax(reached, axis=-1) + 1
    return np.where(reached.any(axis=-1), first, nb).astype(np.int32)


def select_blocks_cdf(q, k, block: int, tau: float, capacity: int,
                      return_scores: bool = False):
    """Stage 1 with the CDF threshold instead of a fixed budget.

    Returns (counts [H, nb] int32, idx [H, nb, capacity] int32).  Row (h, i)
    keeps its top min(counts[h, i], capacity) blocks (by pooled probability,
    ties to the lower index) in ascending order; the rest of the row repeats
    its last kept block, so that idx is also a valid fixed-capacity kept list
    (duplicates name the same block).
    """
    sc = selection_scores(q, k, None, block, 0.0)
    counts = cdf_counts(sc["probs"], tau)
    h_count, nb, _ = sc["probs"].shape
    idx = np.zeros((h_count, nb, capacity), dtype=np.int32)
    order = np.argsort(-sc["probs"], axis=-1, kind="stable")
    for h in range(h_count):
        for i in range(nb):
            keep = min(int(counts[h, i]), capacity)
            kept = np.sort(order[h, i, :keep])
            idx[h, i, :keep] = kept
            idx[h, i, keep:] = kept[-1]
    if return_scores:
        return counts, idx, sc
    return counts, idx


# ---------------------------------------------------------------------------
# Stage 2: block-sparse attention
# ---------------------------------------------------------------------------

def _block_tokens(x_h: np.ndarray, blocks: Sequence[int], block: int) -> np.ndarray:
    return np.concatenate([x_h[j * block:(j + 1) * block] for j in blocks], axis=0)


def sparse_attention_block(q, k, v, kept: Sequence[int], h: int, i: int,
                           block: int) -> Tuple[np.ndarray, np.ndarray]:
    """Attention output and lse of query block ``i`` of head ``h``.

    For each query token n of the block: softmax over the tokens of the kept
    key blocks only of (Q[n] . K[t]) / sqrt(d), weighted sum of V[t]; no causal
    mask (ReSS, Table S5: global attention is bidirectional).  The kept blocks
    are executed exactly (VASC, section 4.2: the mask is passed to the sparse
    kernel).  lse[n] = ln sum_t exp(logit[n, t]) over the kept tokens.
    Returns (O [B, d], lse [B]).
    """
    q_blk = _f64(q[i * block:(i + 1) * block, h, :])
    k_h = _f64(k[:, h, :])
    v_h = _f64(v[:, h, :])
    d = q_blk.shape[-1]
    keys = _block_tokens(k_h, kept, block)
    vals = _block_tokens(v_h, kept, block)
    s = (q_blk @ keys.T) / math.sqrt(d)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    out = (e @ vals) / l
    lse = m[:, 0] + np.log(l[:, 0])
    return out, lse


def sparse_attention(q, k, v, idx, block: int,
                     rows: Optional[Iterable[Tuple[int, int]]] = None):
    """Stage 2 over every (head, query block) row, or over ``rows`` only.

    Returns (O [N, H, d], lse [H, N]) in float64; rows not computed are NaN.
    """
    n, h_count, d = q.shape
    nb = n // block
    out = np.full((n, h_count, d), np.nan)
    lse = np.full((h_count, n), np.nan)
    if rows is None:
        rows = [(h, i) for h in range(h_count) for i in range(nb)]
    for h, i in rows:
        o_blk, lse_blk = sparse_attention_block(q, k, v, idx[h, i], h, i, block)
        out[i * block:(i + 1) * block, h, :] = o_blk
        lse[h, i * block:(i + 1) * block] = lse_blk
    return out, lse


# ---------------------------------------------------------------------------
# Stage 3: drift of the dropped blocks
# ---------------------------------------------------------------------------

def dropped_blocks(kept: Sequence[int], nb: int) -> np.ndarray:
    """Complement of the kept set, ascending."""
    mask = np.ones(nb, dtype=bool)
    mask[np.asarray(kept, dtype=np.int64)] = False
    return np.nonzero(mask)[0]


def drift_block(q, k, v, kept: Sequence[int], lse_blk, h: int, i: int,
                block: int) -> Tuple[np.ndarray, float]:
    """Per-dropped-block drift and drop-set drift J of query block ``i``, head ``h``.

    Masking a key block shifts what attention writes into the residual stream
    (ReSS, Fig. 1 and Fig. 3(a)); the drift score measures that shift per block
    (ReSS, Fig. 3(b)), and the drift of a drop set depends on the directions of
    the contributions, not only their sizes (ReSS, Abstract), so the set drift
    is the norm of their sum (ReSS, Fig. 9 plots quality against it).

    For a dropped block j and query token n of block i:
        C_j[n, :] = sum_{t in block j} exp(logit[n, t] - lse[n]) * V[t, :]
    with lse the kept-set normaliser of stage 2 (reading: the sparse pass's
    lse).  drift_j = ||C_j||_F over the B x d matrix, and
    J = || sum_{j dropped} C_j ||_F.
    Returns (drift over the dropped blocks in ascending j, J).
    """
    q_blk = _f64(q[i * block:(i + 1) * block, h, :])
    k_h = _f64(k[:, h, :])
    v_h = _f64(v[:, h, :])
    n, d = k_h.shape
    nb = n // block
    lse_blk = _f64(lse_blk)
    drop = dropped_blocks(kept, nb)
    nd = drop.shape[0]
    if nd == 0:
        return np.zeros(0), 0.0
    keys = _block_tokens(k_h, drop, block)                      # [nd*B, d]
    vals = _block_tokens(v_h, drop, block).reshape(nd, block, d)
    s = (q_blk @ keys.T) / math.sqrt(d)                          # [Bq, nd*B]
    w = np.exp(s - lse_blk[:, None]).reshape(q_blk.shape[0], nd, block)
    contrib = np.einsum("rnb,nbd->nrd", w, vals)                 # C_j: [nd, Bq, d]
    drift = np.sqrt((contrib * contrib).sum(axis=(1, 2)))
    total = contrib.sum(axis=0)
    return drift, float(np.sqrt((total * total).sum()))


def block_drift(q, k, v, idx, lse, block: int,
                rows: Optional[Iterable[Tuple[int, int]]] = None):
    """Stage 3 over every row, or over ``rows`` only.

    Returns (drift [H, nb, nb - k], J [H, nb]) in float64; rows not computed
    are NaN.
    """
    n, h_count, _ = q.shape
    nb = n // block
    budget = idx.shape[-1]
    drift = np.full((h_count, nb, nb - budget), np.nan)
    jset = np.full((h_count, nb), np.nan)
    if rows is None:
        rows = [(h, i) for h in range(h_count) for i in range(nb)]
    lse = _f64(lse)
    for h, i in rows:
        dr, jv = drift_block(q, k, v, idx[h, i], lse[h, i * block:(i + 1) * block], h, i, block)
        drift[h, i, :] = dr
        jset[h, i] = jv
    return drift, jset


# ---------------------------------------------------------------------------
# Layout-aware variant: padding and the special (camera, register) tokens
# ---------------------------------------------------------------------------

def view_layout(n_tokens: int, tokens_per_view: int, real_tokens_per_view: int,
                n_special: int = 5) -> Tuple[np.ndarray, np.ndarray]:
    """Boolean masks (valid [N], special [N]) of concatenated padded views.

    A VGGT view is 1 camera + 4 register tokens followed by its patch tokens,
    zero-padded to ``tokens_per_view``; positions ``real_tokens_per_view`` ..
    ``tokens_per_view - 1`` of every view are padding, positions 0 ..
    ``n_special - 1`` are the special tokens.
    """
    pos = np.arange(n_tokens) % tokens_per_view
    valid = pos < real_tokens_per_view
    special = valid & (pos < n_special)
    return valid, special


def pool_blocks_valid(x, block: int, valid) -> Tuple[np.ndarray, np.ndarray]:
    """Mean of the valid tokens of each block, per head, and the valid counts.

    Reading: padding does not enter a block's mean; a block without a valid
    token pools to the zero vector and is empty.  Returns (pooled [H, nb, d],
    counts [nb]).
    """
    x = _f64(x)
    valid = np.asarray(valid, dtype=bool)
    n, h, d = x.shape
    nb = n // block
    w = valid.reshape(nb, block).astype(np.float64)
    counts = w.sum(axis=1)
    sums = np.einsum("jb,jbhd->jhd", w, x.reshape(nb, block, h, d))
    pooled = sums / np.maximum(counts, 1.0)[:, None, None]
    return np.ascontiguousarray(pooled.transpose(1, 0, 2)), counts.astype(np.int64)


def select_blocks_layout(q, k, block: int, budget: int, valid, special,
                         return_scores: bool = False):
    """Stage 1 with padding and special tokens (VASC section 4.2: camera and
    register queries stay dense and key blocks made only of special tokens
    are always kept; VASC A.5: the special queries keep dense attention).

    Readings: pooled means over valid tokens only; the pooled logits as in
    ``block_logits``; an empty key block is never preferred to a non-empty
    one; a special-only key block (at least one valid token, all of them
    special) is always kept and counts toward the budget (when there are more
    than ``budget`` of them, the lowest-index ones); the rest of the budget
    goes to the largest logits, ties to the lower index.
    """
    valid = np.asarray(valid, dtype=bool)
    special = np.asarray(special, dtype=bool)
    qbar, _ = pool_blocks_valid(q, block, valid)
    kbar, kcount = pool_blocks_valid(k, block, valid)
    logits = block_logits(qbar, kbar)
    nb = kbar.shape[1]
    sp = (special & valid).reshape(nb, block).sum(axis=1)
    forced = (kcount > 0) & (sp == kcount)
    empty = kcount == 0
    rank = logits.copy()
    rank[:, :, empty] = -np.inf
    rank[:, :, forced] = np.inf
    idx = topk_lowest_index(rank, budget)
    if return_scores:
        return idx, {"logits": logits, "forced": forced, "empty": empty}
    return idx


def sparse_attention_layout_block(q, k, v, kept: Sequence[int], h: int, i: int, block: int,
                                  valid, special) -> Tuple[np.ndarray, np.ndarray]:
    """Stage 2 for query block ``i`` of head ``h`` with padding and special tokens.

    For query token n: a padding query gets output 0 and lse -inf; a special
    query attends densely to every valid key of the sequence; any other query
    attends to the valid tokens of the kept blocks.  Padding keys never enter
    a softmax.  Returns (O [B, d], lse [B]).
    """
    valid = np.asarray(valid, dtype=bool)
    special = np.asarray(special, dtype=bool)
    q_h = _f64(q[:, h, :])
    k_h = _f64(k[:, h, :])
    v_h = _f64(v[:, h, :])
    n, d = k_h.shape
    kept_tok = np.zeros(n, dtype=bool)
    for j in kept:
        kept_tok[j * block:(j + 1) * block] = True
    out = np.zeros((block, d))
    lse = np.full(block, -np.inf)
    for r in range(block):
        t = i * block + r
        if not valid[t]:
            continue
        keys = valid if special[t] else (valid & kept_tok)
        if not keys.any():
            continue
        s = (k_h[keys] @ q_h[t]) / math.sqrt(d)
        m = s.max()
        e = np.exp(s - m)
        out[r] = (e @ v_h[keys]) / e.sum()
        lse[r] = m + np.log(e.sum())
    return out, lse


def drift_layout_block(q, k, v, kept: Sequence[int], lse_blk, h: int, i: int, block: int,
                       valid, special) -> Tuple[np.ndarray, float]:
    """Stage 3 for query block ``i`` of head ``h`` with padding and special tokens.

    As ``drift_block`` over the valid keys of each dropped block, for the
    valid non-special queries of block i; a special query drops nothing and a
    padding query writes nothing, so their rows of every C_j are zero.
    """
    valid = np.asarray(valid, dtype=bool)
    special = np.asarray(special, dtype=bool)
    q_h = _f64(q[:, h, :])
    k_h = _f64(k[:, h, :])
    v_h = _f64(v[:, h, :])
    n, d = k_h.shape
    nb = n // block
    lse_blk = _f64(lse_blk)
    drop = dropped_blocks(kept, nb)
    if drop.shape[0] == 0:
        return np.zeros(0), 0.0
    rows = np.arange(i * block, (i + 1) * block)
    live = valid[rows] & ~special[rows]
    contrib = np.zeros((drop.shape[0], block, d))
    for c, j in enumerate(drop):
        toks = np.arange(j * block, (j + 1) * block)
        toks = toks[valid[toks]]
        if toks.shape[0] == 0:
            continue
        s = (q_h[rows] @ k_h[toks].T) / math.sqrt(d)
        # rows that write nothing (lse -inf for padding) take a finite stand-in
        lse_live = np.where(live, lse_blk, 0.0)
        w = np.exp(s - lse_live[:, None]) * live[:, None]
        contrib[c] = w @ v_h[toks]
    drift = np.sqrt((contrib * contrib).sum(axis=(1, 2)))
    total = contrib.sum(axis=0)
    return drift, float(np.sqrt((total * total).sum()))


# ---------------------------------------------------------------------------
# ReSS: drift-based selection with iterative residual restoration (pooled)
# ---------------------------------------------------------------------------

def pooled_contributions(q, k, v, block: int) -> np.ndarray:
    """c[h, i, j, :] = p[h, i, j] * Vbar[h, j]: what key block j adds to the
    pooled output of query block i, with p the pooled probabilities of
    stage 1.

    ReSS measures the shift each block leaves in the residual stream when it
    is masked (ReSS, Fig. 1 and Fig. 3(a)).  Reading: at block granularity,
    the pooled query of block i attends to key block j with its pooled
    probability, and block j's values enter as their mean, so block j's
    contribution is p_ij * Vbar_j.
    """
    sc = selection_scores(q, k, None, block, 0.0)
    vbar = pool_blocks(v, block)
    return sc["probs"][..., None] * vbar[:, None, :, :]


def drop_set_drift(contrib_row, kept: Sequence[int]) -> float:
    """J(D) = || sum_{j in D} c_j ||_2 over the drop set D (the complement of
    `kept`): the drift of a drop set depends on the directions of the
    contributions, not only on their sizes (ReSS, Abstract)."""
    c = _f64(contrib_row)
    drop = dropped_blocks(kept, c.shape[0])
    return float(np.linalg.norm(c[drop].sum(axis=0)))


def restore_row(contrib_row, budget: int, rounds: int, cand: int = 8):
    """Drift-based selection of one (head, query block) row.

    1. Drift score d_j = ||c_j||_2; the initial kept set is the `budget`
       blocks of largest drift score, ties to the lower index (ReSS, Fig. 3(b):
       the blocks with the highest scores form the initial selected set).
    2. Up to `rounds` restoration rounds, each one budget-preserving swap that
       reduces the drift J of the drop set (ReSS, Fig. 3(c)).  Reading of the
       swap rule (the pages do not give it): with T = sum_{j in D} c_j,
         - the candidates to restore (leave D) are the `cand` dropped blocks of
           largest gain 2 <T, c_b> - ||c_b||^2 (ties: lower index),
         - the candidates to drop (enter D) are the `cand` kept blocks of
           smallest cost 2 <T, c_a> + ||c_a||^2 (ties: lower index),
         - among those pairs the one of smallest ||T - c_b + c_a|| is taken
           (ties: lower b, then lower a), and the round swaps a and b if that
           is strictly below J; otherwise restoration stops.
    3. Track-best: the kept set of smallest J over the initial set and every
       round (ReSS, Table S3).  Every accepted swap lowers J, so it is the
       last one.
    Returns (kept blocks ascending, J of the initial set, J of the result).
    """
    c = _f64(contrib_row)
    nb = c.shape[0]
    score = np.sqrt((c * c).sum(axis=1))
    order = np.argsort(-score, kind="stable")
    kept = set(order[:budget].tolist())
    j0 = drop_set_drift(c, sorted(kept))
    best = (j0, sorted(kept))
    for _ in range(rounds):
        drop = [j for j in range(nb) if j not in kept]
        if not drop or not kept:
            break
        t = c[drop].sum(axis=0)
        jcur = float(np.linalg.norm(t))
        gain = {b: 2.0 * (t @ c[b]) - c[b] @ c[b] for b in drop}
        cost = {a: 2.0 * (t @ c[a]) + c[a] @ c[a] for a in kept}
        out = sorted(drop, key=lambda b: (-gain[b], b))[:cand]
        inn = sorted(kept, key=lambda a: (cost[a], a))[:cand]
        pairs = sorted(((float(np.linalg.norm(t - c[b] + c[a])), b, a) for b in out for a in inn))
        jnew, b, a = pairs[0]
        if not jnew < jcur:
            break
        kept.remove(a)
        kept.add(b)
        if jnew < best[0]:
            best = (jnew, sorted(kept))
    return np.asarray(best[1], dtype=np.int32), j0, best[0]


def select_blocks_restore(q, k, v, block: int, budget: int, rounds: int, cand: int = 8):
    """ReSS-style selection of every row: idx [H, nb, budget] int32 ascending,
    and J [H, nb] of the initial and of the restored drop sets."""
    contrib = pooled_contributions(q, k, v, block)
    h_count, nb = contrib.shape[:2]
    idx = np.zeros((h_count, nb, budget), dtype=np.int32)
    j_init = np.zeros((h_count, nb))
    j_final = np.zeros((h_count, nb))
    for h in range(h_count):
        for i in range(nb):
            idx[h, i], j_init[h, i], j_final[h, i] = restore_row(contrib[h, i], budget, rounds, cand)
    return idx, j_init, j_final


# ---------------------------------------------------------------------------
# VASC: value-aware demand, budgeted binary execution, cross-layer memory
# ---------------------------------------------------------------------------

def block_pairs(nb: int) -> Tuple[np.ndarray, np.ndarray]:
    """Fixed pairs of adjacent key blocks in native order.

    VASC A.1: neighbouring children in native order form fixed pairs, and an
    unpaired final child is a singleton.  Returns (pair_of [nb]: the pair of
    each block, size [n_pairs]: 2, or 1 for a final singleton).
    """
    pair_of = np.arange(nb) // 2
    n_pairs = (nb + 1) // 2
    size = np.full(n_pairs, 2, dtype=np.int64)
    if nb % 2 == 1:
        size[-1] = 1
    return pair_of, size


def pair_contrast(vbar) -> np.ndarray:
    """rho[h, p]: the RMS contrast of the pooled values of pair p.

    VASC 4.1 and A.3: the two children of a pair share one contrast signal,
    the root mean square over the head dimension of the difference of their
    pooled values; a singleton is paired with itself, so its contrast is 0.
        rho[h, p] = sqrt( (1/d) * sum_d (Vbar[h, 2p, d] - Vbar[h, 2p+1, d])^2 )
    """
    vbar = _f64(vbar)
    h, nb, d = vbar.shape
    n_pairs = (nb + 1) // 2
    rho = np.zeros((h, n_pairs), dtype=np.float64)
    for p in range(nb // 2):
        diff = vbar[:, 2 * p, :] - vbar[:, 2 * p + 1, :]
        rho[:, p] = np.sqrt((diff * diff).sum(axis=-1) / d)
    return rho


def vasc_demand(probs, rho, budgets, value_aware: bool = True) -> np.ndarray:
    """Current demand a[h, i, j] of every (head, query block, key block).

    VASC 4.1: the pair's contrast modulates the query's relevance, and the
    demand is rescaled and clipped to the query's capacity; A.2: every entry
    is at most one and the row's total at most the capacity.  Readings:
      * relevance is the pooled probability p_ij, modulated by multiplying
        with the contrast of j's pair (with value_aware False the contrast
        is one: the ablation that sets the paired-value contrast to one,
        VASC Appendix D);
      * the rescaling is proportional to the row's capacity c_h (ReSS Fig. 3
        and Table 2 give each head its own budget c_h) and the clip is
        applied once:
            d_ij = p_ij * rho[h, pair(j)]
            a_ij = min(1, c_h * d_ij / sum_j d_ij)   (0 when the sum is 0).
    """
    p = _f64(probs)
    h_count, nbq, nb = p.shape
    pair_of, _ = block_pairs(nb)
    if value_aware:
        factor = _f64(rho)[:, pair_of]                    # [H, nb]
    else:
        factor = np.ones((h_count, nb), dtype=np.float64)
    a = np.zeros_like(p)
    for h in range(h_count):
        c = float(budgets[h])
        for i in range(nbq):
            d = p[h, i] * factor[h]
            total = d.sum()
            if total > 0.0:
                a[h, i] = np.minimum(1.0, c * d / total)
    return a


def memory_ranking_copy(memory) -> np.ndarray:
    """The copy of the pair memory that enters the ranking.

    VASC A.4: normalisation runs per batch entry and head and only on the
    ranking copy (the raw balance is carried on unchanged); 4.3: the copy is
    bounded.  Reading: divide each head's balances by their largest value, so
    the copy lies in [0, 1] (all zero when the head has no deficit).
    """
    m = _f64(memory)
    out = np.zeros_like(m)
    for h in range(m.shape[0]):
        top = m[h].max() if m.shape[1] else 0.0
        if top > 0.0:
            out[h] = m[h] / top
    return out


def pair_means(x) -> np.ndarray:
    """mean over query blocks i and the children j of pair p of x[h, i, j].

    VASC 4.3: demand and service are averaged over query blocks and paired
    children; A.3: a singleton is averaged over its one child.
    """
    x = _f64(x)
    h_count, nbq, nb = x.shape
    pair_of, size = block_pairs(nb)
    out = np.zeros((h_count, size.shape[0]), dtype=np.float64)
    for j in range(nb):
        out[:, pair_of[j]] += x[:, :, j].sum(axis=1)
    return out / (nbq * size)[None, :]


def select_blocks_vasc(q, k, v, block: int, budgets, capacity: int, memory=None,
                       value_aware: bool = True):
    """One global layer of VASC's selection and its memory settlement.

    1. pooled probabilities p (as ``selection_scores`` with lam = 0) and the
       pair contrast rho of the pooled values;
    2. the current demand a (``vasc_demand``);
    3. the ranking score a_ij + M[h, pair(j)], M the ranking copy of the
       memory carried in (VASC 4.2: memory augments the current demand;
       reading: it is added);
    4. a binary mask of exactly c_h blocks per row (VASC 4.2 and A.2), the
       largest scores, ties to the lower index;
    5. the settlement (VASC 4.3 and A.5): with D and S the pair means of the
       demand and of the executed mask,
           memory_out = max(0, memory_in + D - S)
       (the accumulated deficit is clipped at zero; no memory, i.e. the
       first layer of an inference, is all zero).

    ``budgets`` holds c_h per head, 1 <= c_h <= capacity.  Returns (idx
    [H, nb, capacity] int32: the c_h kept blocks ascending, then the last of
    them repeated; memory_out [H, n_pairs]; a dict with probs, rho, demand,
    mhat, score, mask, D and S).
    """
    sc = selection_scores(q, k, None, block, 0.0)
    probs = sc["probs"]
    h_count, nbq, nb = probs.shape
    _, size = block_pairs(nb)
    if value_aware:
        assert v is not None, "the value contrast needs V"
        rho = pair_contrast(pool_blocks(v, block))
    else:
        rho = np.ones((h_count, size.shape[0]), dtype=np.float64)   # unused: contrast one
    mem_in = np.zeros((h_count, size.shape[0])) if memory is None else _f64(memory)
    demand = vasc_demand(probs, rho, budgets, value_aware)
    mhat = memory_ranking_copy(mem_in)
    pair_of, _ = block_pairs(nb)
    score = demand + mhat[:, None, pair_of]
    idx = np.zeros((h_count, nbq, capacity), dtype=np.int32)
    mask = np.zeros_like(score)
    for h in range(h_count):
        c = int(budgets[h])
        kept = topk_lowest_index(score[h], c)            # [nbq, c] ascending
        idx[h, :, :c] = kept
        idx[h, :, c:] = kept[:, -1:]
        for i in range(nbq):
            mask[h, i, kept[i]] = 1.0
    dmean = pair_means(demand)
    smean = pair_means(mask)
    mem_out = np.maximum(0.0, mem_in + dmean - smean)
    info = {"probs": probs, "rho": rho, "demand": demand, "mhat": mhat, "score": score,
            "mask": mask, "D": dmean, "S": smean}
    return idx, mem_out, info
