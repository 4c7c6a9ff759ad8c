"""Plain fp64 CPU oracle for query-dependent block-sparse causal attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module: only the tests, the
smoke check in ``__graft_entry__`` and the ``cpu_baseline`` / ``--impl reference`` legs of the
benchmark may call it.  It shares no code with the CUDA library.  It is deliberately slow: every
function is the plain definition, one query (or one block) at a time, in float64, with NumPy only
for array storage, matrix-vector products and sums.

Sources (cited by page title and the section / equation on it):

* [SAS] the review page "SAS: Simple Attention Sparsification via End-to-End Optimization of
  Context Ranking" -- sections "Background: the problem they solved" (Eq. 1-3), "The new
  approach: SAS" (Eq. 4, Eq. 9), "Why the four design choices matter" (Eq. 5 and the softmax gate
  log g = s - LSE(s)), "How it works: a worked example" (steps 1-6), "Decoding efficiency"
  (Fig. 7).
* [FreeSolo] the summary page "FreeSolo가 학습 길이의 64배까지 제로샷 검색을 유지한다" --
  section "How it works" (cells, the three summaries, the query-block prefix, the erf-biased cell
  score, top-K cells, the RoPE sliding-window branch, the NoPE long branch, the per-head mix)
  and section "How it differs" (the FS-L variant: W recent cells plus the P largest key norms,
  pruned before the query arrives, a fixed-size state; the FS-B variant: two forests per head
  searched by a beam with node upper bounds, log-sum-exp re-rank over token keys).
* [Monodratic] the article "Monodratic、学習ルーティングによりスパース因果アテンションの選択性を高め
  られると主張" -- section on turning sparse attention into a retrieval decision (guaranteed local
  block, exact causal softmax over the selected tokens, no future block reachable, sparse-vs-dense
  mask parity).

Readings where the pages are silent or garbled (the numbering is that of the design notes):

* R1 gate normaliser: log g_m = s_m - LSE over either the selected history blocks
  ("selected") or every history block ("all"); the worked example of [SAS] uses all blocks.
* R2 GQA: query head h reads kv head h // (Hq // Hk); selection is per query head.
* R3 current block of the query at position i is cur = i // b; history blocks are 0 .. cur-1.
* R4 fewer candidates than K: all candidates are taken.  FreeSolo queries with no candidate cell
  use the short branch alone.
* R5 top-K order: larger score first, lower block index first among equal scores, NaN below
  everything; the result is reported in ascending block order.
* R6 logits and dot-product scores use the scale 1/sqrt(d).
* R7 block centre = mean position of the tokens in the block (c*b + (b-1)/2 for a full block).
* R8 FreeSolo mix o = (1 - alpha_h) * o_short + alpha_h * o_long; RoPE with base 10000,
  rotate-half pairing, absolute positions; the window holds the ``window`` most recent keys,
  the query's own key included.
* R9 erf argument (i - p_c) / (2 sigma_h), as printed, positive for past cells.
* R10 dg is the derivative with respect to g_m (not log g_m), one value per (query unit, selected
  history block); with per-query-block selection it sums over the unit's queries.
* R11 a computed selector score is rounded to float32 before top-K, the precision in which the
  CUDA kernels take the same decision; supplied scores are float32 already.
* R20 outer gate (f1 variant): the gate multiplies the value contributions of its block outside
  the softmax, o = sum_j g_m(j) p_j v_j with p the ungated softmax; the current block has gate 1;
  g = softmax of the scores over the normaliser set, as for the inner gate.
* R21 FS-B (the pages name the forests' contents, the beam width and the re-rank but not the tree
  shape): per head one forest over every candidate cell and one over the ceil(n/2) cells of
  largest key norm; a forest is a row of perfect binary trees over consecutive cells in position
  order (one per set bit of the cell count); a node keeps the mean of its leaves' mean keys, the
  largest distance of a leaf mean key from it (radius), the largest leaf norm and the smallest
  leaf centre; the beam ranks nodes by the Cauchy-Schwarz bound built from those four values.
* R19 GQA-shared selection (a variant; the pages leave per-head versus shared selection open):
  the group's score of a block is the mean of its query heads' scores, its top-K is attended by
  every head of the group; bf16 summaries are the float32 mean keys rounded to the nearest
  bfloat16 (ties to even).
"""
from __future__ import annotations

import itertools
import math

import numpy as np
from scipy.special import erf as _erf

NEG_INF = -math.inf

# ----------------------------------------------------------------------------------------------
# Block partition and summaries
# ----------------------------------------------------------------------------------------------


def block_range(c: int, n: int, b: int) -> tuple[int, int]:
    """Token range [lo, hi) of block c when n positions are cut into blocks of b tokens.

    [SAS] "Background", Eq. 3: the n context positions form C = n / b blocks B_1..B_C of b tokens.
    A final block shorter than b (n not a multiple of b) keeps the remaining tokens.
    """
    return c * b, min(n, (c + 1) * b)


def num_blocks(n: int, b: int) -> int:
    return (n + b - 1) // b


def block_summaries(k: np.ndarray, b: int):
    """Per-block key summaries of one (batch, kv head): mean key, max key norm, centre.

    [FreeSolo] "How it works": each cell keeps its mean key (content used for routing), its
    centre position (for the relative distance) and the largest key norm inside it (a
    query-independent priority).  [SAS] "Limitations" names its summary a pooled block summary.
    Returns mean_k [C, d], max_norm [C], centre [C] in float64.
    """
    k = np.asarray(k, dtype=np.float64)
    n, d = k.shape
    C = num_blocks(n, b)
    mean_k = np.zeros((C, d))
    max_norm = np.zeros(C)
    centre = np.zeros(C)
    for c in range(C):
        lo, hi = block_range(c, n, b)
        blk = k[lo:hi]
        mean_k[c] = blk.sum(axis=0) / (hi - lo)
        max_norm[c] = max(math.sqrt(float(np.dot(row, row))) for row in blk)
        centre[c] = sum(range(lo, hi)) / (hi - lo)  # R7: mean token position
    return mean_k, max_norm, centre


# ----------------------------------------------------------------------------------------------
# Block scoring
# ----------------------------------------------------------------------------------------------


def dot_scores(q: np.ndarray, mean_k: np.ndarray, n_cand: int) -> np.ndarray:
    """s_c = q . kbar_c / sqrt(d) for the n_cand candidate blocks (c < n_cand).

    First term of the cell score r_ic of [FreeSolo] "How it works"; the plain query-summary score
    a learned selector is replaced by when no selector weights exist.  R6.
    """
    q = np.asarray(q, dtype=np.float64)
    d = q.shape[0]
    return np.array([float(np.dot(q, mean_k[c])) / math.sqrt(d) for c in range(n_cand)])


def freesolo_scores(q, i, mean_k, max_norm, centre, lam, sigma, n_cand) -> np.ndarray:
    """r_ic = q_i . kbar_c / sqrt(d) + lambda_h * a_c * erf((i - p_c) / (2 sigma_h)).

    [FreeSolo] "How it works", the cell score.  ``erf`` is the library error function.  R9.
    """
    base = dot_scores(q, mean_k, n_cand)
    bias = np.array([lam * max_norm[c] * float(_erf((i - centre[c]) / (2.0 * sigma)))
                     for c in range(n_cand)])
    return base + bias


def sas_num_candidates(i: int, b: int) -> int:
    """History blocks available to the query at position i: blocks 0 .. cur-1, cur = i // b.

    [SAS] "The new approach", Eq. 4: the selector scores only history blocks; the current block
    B_0 is always kept outside the selection.  R3.
    """
    return i // b


def freesolo_num_candidates(i: int, cell: int, q_block: int) -> int:
    """Cells whose tokens all lie before the start of the query's block of q_block queries.

    [FreeSolo] "How it works": the prefix is fixed per query block (B = 128), so every query of
    one block sees the same candidate cells: those ending at or before floor(i / B) * B.
    """
    prefix = (i // q_block) * q_block
    return prefix // cell


# ----------------------------------------------------------------------------------------------
# Top-K selection
# ----------------------------------------------------------------------------------------------


def _rank_key(value: float, idx: int):
    """Sort key: NaN last, then larger score first, then lower index first (R5)."""
    if math.isnan(value):
        return (1, 0.0, idx)
    return (0, -value, idx)


def topk_blocks(s, n_cand: int, K: int) -> list[int]:
    """Indices of the K highest-scoring candidate blocks c < n_cand, in ascending order.

    [SAS] "Background", Eq. 3 (I = Top-K(s, K)) and "How it works" step 3; fewer than K candidates
    are all taken (R4).  A full stable sort over the candidates decides the set.
    """
    order = sorted(range(n_cand), key=lambda c: _rank_key(float(s[c]), c))
    return sorted(order[:min(K, n_cand)])


def fsl_candidates(max_norm, n_cells: int, W: int, P: int) -> list[int]:
    """FS-L pre-query pruning: the cells a head keeps before any query arrives.

    [FreeSolo] "How it differs" (FS-L): each head keeps its W most recent cells and the
    P cells of largest maximum key norm, and queries pick their top K inside that set.  R18: the
    P cells are taken among the cells older than the W recent ones (the two parts are disjoint),
    larger norm first, lower index on ties, NaN last; fewer cells than W + P are all kept.
    Returns ascending cell indices among c < n_cells.
    """
    recent = list(range(max(0, n_cells - W), n_cells))
    older = n_cells - len(recent)
    return sorted(topk_blocks(max_norm, older, P) + recent)


def fsl_select(q, i, mean_k, max_norm, centre, lam, sigma, cand, K) -> list[int]:
    """Top-K of the FreeSolo cell score over the pruned candidates only (ascending cells).

    [FreeSolo] "How it differs" (FS-L) with the cell score of "How it works": the FS-L query
    scores the kept cells with the same r_ic as the full method and reads its K best.  R18 tie
    rule: larger score, then lower cell index.
    """
    cand = [int(c) for c in cand]
    if not cand:
        return []
    r = freesolo_scores(q, i, mean_k, max_norm, centre, lam, sigma, max(cand) + 1)
    order = sorted(cand, key=lambda c: _rank_key(float(round_f32(r[c])), c))
    return sorted(order[:min(K, len(cand))])


def _outranks(a, x: int, y: int) -> bool:
    """Cell x ranks above cell y by maximum key norm (larger first, lower index on ties, NaN last)."""
    return _rank_key(float(a[x]), x) < _rank_key(float(a[y]), y)


def fsl_state_new(W: int, P: int) -> dict:
    """An empty FS-L state: no candidate cell yet ([FreeSolo] "How it differs", FS-L: the state a
    head keeps has a fixed size, W recent cells plus P cells chosen by key norm)."""
    return {"W": W, "P": P, "n_cells": 0, "older": []}


def fsl_state_advance(state: dict, max_norm, n_cells: int) -> dict:
    """Grow the candidate prefix of an FS-L state to ``n_cells`` cells, one cell at a time.

    [FreeSolo] "How it differs" (FS-L): the pruning happens before the query arrives and the state
    stays W + P cells.  R18 as an update rule: the W newest candidate cells are kept outright; when
    a cell drops out of them it joins the older cells, of which the state keeps the P best by
    maximum key norm (larger first, lower index on ties, NaN last).  The joining cell has the
    highest index of all older cells, so it enters only if it strictly outranks the lowest-ranked
    kept older cell (which it then replaces), or if fewer than P are kept.  Each step looks at
    the P kept cells only, never at the whole prefix.
    """
    W, P = state["W"], state["P"]
    older = list(state["older"])
    for m in range(state["n_cells"] + 1, n_cells + 1):  # the prefix grows to m cells
        c = m - 1 - W  # the cell leaving the W newest
        if c < 0 or P == 0:
            continue
        if len(older) < P:
            older.append(c)
            continue
        worst = older[0]
        for x in older[1:]:
            if _outranks(max_norm, worst, x):
                worst = x
        if _outranks(max_norm, c, worst):
            older.remove(worst)
            older.append(c)
    return {"W": W, "P": P, "n_cells": max(n_cells, state["n_cells"]), "older": older}


def fsl_state_cells(state: dict) -> list[int]:
    """The cells an FS-L state keeps: its older cells and the W newest, ascending."""
    n, W = state["n_cells"], state["W"]
    return sorted(state["older"]) + list(range(max(0, n - W), n))


def fsl_decode_row(q, k, v, i, summaries, cand, cell, K, window, lam, sigma, alpha, theta):
    """FS-L decode output of the query at position i of one head: the two branches of the full
    method ([FreeSolo] "How it works": RoPE window, NoPE long branch, per-head mix) with the long
    branch's cells chosen among the state's kept cells ``cand`` only ([FreeSolo] "How it
    differs", FS-L: the query takes its top K inside the pruned set)."""
    mean_k, max_norm, centre = summaries
    sel = fsl_select(q, i, mean_k, max_norm, centre, lam, sigma, cand, K)
    o, _ = freesolo_row(q, k, v, i, summaries, cell, 128, K, window, lam, sigma, alpha, theta,
                        selection=sel)
    return o, sel


def round_f32(x):
    """R11: the precision in which a computed score decides the selection."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def round_bf16(x):
    """Nearest bfloat16 of each float32 value, ties to the even significand; NaN stays NaN (R19).

    bfloat16 keeps the sign, the 8 exponent bits and the top 7 fraction bits of a float32.  The
    16 dropped bits decide: above half of the last kept bit rounds the magnitude up, below half
    truncates, exactly half rounds to the even kept pattern (a carry may reach the exponent,
    overflowing to infinity as IEEE rounding does).
    """
    x32 = np.asarray(x, dtype=np.float32)
    u = x32.view(np.uint32).astype(np.uint64)
    kept, dropped = u >> 16, u & 0xFFFF
    up = (dropped > 0x8000) | ((dropped == 0x8000) & ((kept & 1) == 1))
    out = ((kept + up.astype(np.uint64)) << 16).astype(np.uint32).view(np.float32)
    return np.where(np.isnan(x32), np.float32(np.nan), out).astype(np.float64)


def shared_block_scores(per_head_scores) -> np.ndarray:
    """Group score of every block for GQA-shared selection (R19): the mean over the group's
    query heads of their block scores ([G, n_cand] -> [n_cand])."""
    return np.asarray(per_head_scores, dtype=np.float64).mean(axis=0)


def decode_reference_shared(q, k, v, seq_lens, b, K, summaries=None):
    """Decode step with one selection per (batch, kv head) (R19).

    For every kv group: the query heads' scores q . kbar / sqrt(d) over the history blocks, their
    mean (shared_block_scores, rounded to float32 as a decision precision, R11), its top-K, and
    for every head of the group the exact softmax over the selected blocks plus the current one.
    ``summaries`` maps (bi, kh) to (mean_k, ...) to use instead of the fp64 block means.
    Returns dict (bi, h) -> {"idx", "scores", "o", "lse"}.
    """
    B, Hq, d = q.shape
    Hk = k.shape[1]
    G = Hq // Hk
    out = {}
    for bi in range(B):
        L = int(seq_lens[bi])
        i = L - 1
        nc = sas_num_candidates(i, b)
        for kh in range(Hk):
            kk = k[bi, kh, :L]
            vv = v[bi, kh, :L]
            mean_k = (summaries[(bi, kh)] if summaries is not None else block_summaries(kk, b))[0]
            per_head = [dot_scores(q[bi, kh * G + g], mean_k, nc) for g in range(G)]
            s = round_f32(shared_block_scores(per_head))
            sel = topk_blocks(s, nc, K)
            for g in range(G):
                h = kh * G + g
                o, lse = sparse_attention_row(q[bi, h], kk, vv, i, b, sel)
                out[(bi, h)] = {"idx": sel, "scores": s, "o": o, "lse": lse}
    return out


# ----------------------------------------------------------------------------------------------
# Softmax log-gate
# ----------------------------------------------------------------------------------------------


def logsumexp(x) -> float:
    x = np.asarray(x, dtype=np.float64)
    if x.size == 0:
        return NEG_INF
    m = float(np.max(x))
    if m == NEG_INF:
        return NEG_INF
    return m + math.log(float(np.sum(np.exp(x - m))))


def log_gates(s, n_cand: int, selected, norm: str) -> dict[int, float]:
    """log g_m = s_m - LSE(s) for each selected history block m.

    [SAS] "Why the four design choices matter": the softmax gate gives log g_m = s_m - LSE(s);
    "The new approach", Eq. 4: the current block keeps g_0 = 1.  ``norm`` picks the set the LSE
    runs over (R1): "all" = every history block c < n_cand, "selected" = the selected ones.
    """
    s = np.asarray(s, dtype=np.float64)
    if norm == "all":
        L = logsumexp(s[:n_cand])
    elif norm == "selected":
        L = logsumexp(s[list(selected)]) if len(selected) else 0.0
    else:
        raise ValueError(norm)
    return {int(m): float(s[m]) - L for m in selected}


# ----------------------------------------------------------------------------------------------
# Exact softmax over the gathered tokens
# ----------------------------------------------------------------------------------------------


def token_set(i: int, b: int, selected, n: int, keep_current: bool = True):
    """Tokens a query at position i attends: every token of the selected history blocks and the
    tokens j <= i of its current block.

    [SAS] "Background", Eq. 2 (attention restricted to the selected set S) and "How it works"
    step 3 (S = B_0 united with the selected blocks); [Monodratic] (guaranteed local block plus the
    selected remote blocks, causal mask applied inside the selected set).  Returns (tokens,
    owning block of each token).
    """
    toks, owner = [], []
    for m in sorted(selected):
        lo, hi = block_range(m, n, b)
        for j in range(lo, hi):
            if j <= i:  # history blocks lie wholly before i; kept for safety of the definition
                toks.append(j)
                owner.append(m)
    if keep_current:
        cur = i // b
        lo, _ = block_range(cur, n, b)
        for j in range(lo, i + 1):
            toks.append(j)
            owner.append(-1)  # -1 marks the current block
    return np.array(toks, dtype=np.int64), np.array(owner, dtype=np.int64)


def attend(q, k, v, toks, bias):
    """Exact softmax attention of one query over the listed tokens.

    z_j = q . k_j / sqrt(d) + bias_j; p = softmax(z); o = sum_j p_j v_j; lse = log sum_j exp z_j.
    [SAS] "Background", Eq. 1-2 (standard attention restricted to S), R6.  Returns o, lse, p.
    """
    q = np.asarray(q, dtype=np.float64)
    d = q.shape[0]
    kk = np.asarray(k[toks], dtype=np.float64)
    vv = np.asarray(v[toks], dtype=np.float64)
    z = kk @ q / math.sqrt(d) + bias
    m = float(np.max(z))
    e = np.exp(z - m)
    l = float(np.sum(e))
    p = e / l
    o = p @ vv
    return o, m + math.log(l), p


def sparse_attention_row(q, k, v, i, b, selected, gate=None, keep_current=True):
    """Output and log-sum-exp of one query at position i over its gathered token set.

    Without a gate this is the inference path of [SAS] "How it works" step 6 (plain Top-K, exact
    softmax over the kept blocks).  With ``gate`` (a dict m -> log g_m) it is the training-mode
    forward of [SAS] "The new approach", Eq. 9: log g_m is added to the logits of every token of
    selected history block m, the current block gets log 1 = 0.
    """
    n = k.shape[0]
    toks, owner = token_set(i, b, selected, n, keep_current)
    bias = np.zeros(len(toks))
    if gate is not None:
        for t, m in enumerate(owner):
            if m >= 0:
                bias[t] = gate[int(m)]
    o, lse, _ = attend(q, k, v, toks, bias)
    return o, lse


def outer_gated_row(q, k, v, i, b, selected, g):
    """Outer-gate forward of one query ([SAS] "Why the four design choices matter", the gate
    placed outside the softmax, R20): p = softmax of the ungated logits over the token set,
    o = sum_j g_m(j) p_j v_j with g_m the gate of history block m (a dict m -> g_m) and 1 for the
    current block; lse is the log-sum-exp of the ungated logits.
    """
    n = k.shape[0]
    toks, owner = token_set(i, b, selected, n)
    _, lse, p = attend(q, k, v, toks, np.zeros(len(toks)))
    w = np.array([p[t] * (g[int(m)] if m >= 0 else 1.0) for t, m in enumerate(owner)])
    o = w @ np.asarray(v[toks], dtype=np.float64)
    return o, lse


def gate_grad_rows_outer(qs, k, v, positions, b, selected, douts):
    """dg_m of the outer gate, summed over the given queries (R20):
        dg_m = sum_{i} sum_{j in B_m} p_ij do_i^T v_j,
    p the ungated softmax of query i over its token set (the gate multiplies the values only, so
    the derivative of o_i with respect to g_m is sum_{j in B_m} p_ij v_j).  Returns dict m -> dg_m.
    """
    n = k.shape[0]
    dg = {int(m): 0.0 for m in selected}
    for q, i, do in zip(qs, positions, douts):
        toks, owner = token_set(int(i), b, selected, n)
        _, _, p = attend(q, k, v, toks, np.zeros(len(toks)))
        do = np.asarray(do, dtype=np.float64)
        for t, m in enumerate(owner):
            if m >= 0:
                dg[int(m)] += p[t] * float(np.dot(do, np.asarray(v[toks[t]], dtype=np.float64)))
    return dg


def masked_attention_row(q, k, v, i, b, selected, gate=None, keep_current=True):
    """The same quantity written as dense attention over all n keys with a -inf mask.

    Independent restatement used to pin the gather path: [Monodratic] compares its sparse
    selected-set attention against an independently built dense mask oracle.
    """
    q = np.asarray(q, dtype=np.float64)
    n, d = k.shape
    z = np.asarray(k, dtype=np.float64) @ q / math.sqrt(d)
    allowed = np.zeros(n, dtype=bool)
    bias = np.zeros(n)
    for m in selected:
        lo, hi = block_range(m, n, b)
        allowed[lo:hi] = True
        if gate is not None:
            bias[lo:hi] = gate[int(m)]
    if keep_current:
        lo, _ = block_range(i // b, n, b)
        allowed[lo:i + 1] = True
    allowed[i + 1:] = False
    z = np.where(allowed, z + bias, NEG_INF)
    w = np.exp(z - z.max())
    w /= w.sum()
    return w @ np.asarray(v, dtype=np.float64)


# ----------------------------------------------------------------------------------------------
# Closed-form gate gradient
# ----------------------------------------------------------------------------------------------


def gate_grad_rows(qs, k, v, positions, b, selected, gate, douts):
    """dg_m for each selected history block m, summed over the given queries.

    [SAS] "Why the four design choices matter", Eq. 5 (inner gate):
        dg_m = sum_{i in B_m} (ptilde_i / g_m) * do^T (v_i - o),
    where ptilde is the gated softmax of the query over its token set and o its output.  The
    queries of one unit share one gate vector, so their contributions add (R10).
    Returns dict m -> dg_m.
    """
    n = k.shape[0]
    dg = {int(m): 0.0 for m in selected}
    for q, i, do in zip(qs, positions, douts):
        toks, owner = token_set(int(i), b, selected, n)
        bias = np.array([gate[int(m)] if m >= 0 else 0.0 for m in owner])
        o, _, p = attend(q, k, v, toks, bias)
        do = np.asarray(do, dtype=np.float64)
        for t, m in enumerate(owner):
            if m < 0:
                continue
            g_m = math.exp(gate[int(m)])
            vi = np.asarray(v[toks[t]], dtype=np.float64)
            dg[int(m)] += p[t] / g_m * float(np.dot(do, vi - o))
    return dg


def selector_grad_row(s, n_cand: int, selected, dg, norm: str):
    """ds_c = dL/ds_c for every history block c < n_cand, from dg_m = dL/dg_m of the selected.

    [SAS] "Why the four design choices matter": log g_m = s_m - LSE(s) over the normaliser set
    (R1), g_m = exp(log g_m).  By the chain rule, dL/dlog g_m = g_m dg_m and
    dlog g_m / ds_c = [c = m] - pi_c, with pi the softmax of s over the normaliser set (0 outside
    it), so ds_c = sum over selected m of g_m dg_m ([c = m] - pi_c).  Returns an array of n_cand.
    """
    s = np.asarray(s, dtype=np.float64)
    sel = [int(m) for m in selected]
    lg = log_gates(s, n_cand, sel, norm)
    if norm == "all":
        norm_set = list(range(n_cand))
    else:
        norm_set = sel
    L = logsumexp(s[norm_set]) if norm_set else 0.0
    pi = np.zeros(n_cand)
    for c in norm_set:
        pi[c] = math.exp(float(s[c]) - L)
    ds = np.zeros(n_cand)
    for m in sel:
        w = math.exp(lg[m]) * float(dg[m])
        for c in range(n_cand):
            ds[c] += w * ((1.0 if c == m else 0.0) - pi[c])
    return ds


def gated_loss(qs, k, v, positions, b, selected, g, douts) -> float:
    """L = sum_i do_i . o_i(g) for gates g (dict m -> g_m > 0); used for finite differences."""
    gate = {m: math.log(gm) for m, gm in g.items()}
    total = 0.0
    for q, i, do in zip(qs, positions, douts):
        o, _ = sparse_attention_row(q, k, v, int(i), b, selected, gate)
        total += float(np.dot(np.asarray(do, dtype=np.float64), o))
    return total


# ----------------------------------------------------------------------------------------------
# Whole-call drivers (decode and prefill), written on top of the row functions
# ----------------------------------------------------------------------------------------------


def decode_reference(q, k, v, seq_lens, b, K, scores=None, gate_norm=None, rows=None,
                     summaries=None):
    """One decode step for every (batch, query head) row, or for the listed ``rows``.

    Chain of [SAS] "How it works" step 6 / the inference algorithm: score the history blocks of
    the query at position seq_len-1 (supplied ``scores`` [B, Hq, C], else q . kbar / sqrt(d)),
    take Top-K, keep the current block, exact softmax over the gathered tokens.  ``gate_norm``
    ("selected" / "all") adds the training-mode log-gate of the supplied or computed scores.
    Returns dict (bi, h) -> {"idx", "scores", "o", "lse"}.
    """
    B, Hq, d = q.shape
    Hk = k.shape[1]
    G = Hq // Hk
    out = {}
    if rows is None:
        rows = [(bi, h) for bi in range(B) for h in range(Hq)]
    cache = {} if summaries is None else summaries
    for bi, h in rows:
        kh = h // G
        L = int(seq_lens[bi])
        i = L - 1
        kk = k[bi, kh, :L]
        vv = v[bi, kh, :L]
        nc = sas_num_candidates(i, b)
        if scores is not None:
            s = np.asarray(scores[bi, h, :nc], dtype=np.float64)
        else:
            if (bi, kh) not in cache:
                cache[(bi, kh)] = block_summaries(kk, b)
            mean_k = cache[(bi, kh)][0]
            s = round_f32(dot_scores(q[bi, h], mean_k, nc))
        sel = topk_blocks(s, nc, K)
        gate = log_gates(s, nc, sel, gate_norm) if gate_norm else None
        o, lse = sparse_attention_row(q[bi, h], kk, vv, i, b, sel, gate)
        out[(bi, h)] = {"idx": sel, "scores": s, "o": o, "lse": lse}
    return out


def prefill_unit_reference(q, k, v, scores, b, q_block, K, bi, h, u, gate_norm=None,
                           dout=None):
    """Prefill of one query unit (query block u of head h): selection shared by the unit.

    The unit's candidates are the history blocks of its first query (c < (u*q_block) // b), its
    selection is Top-K of the supplied scores ``scores[bi, h, u]``; each query i of the unit keeps
    its own current block i // b with the causal mask j <= i ([SAS] "The new approach", Eq. 9 and
    the training forward it describes).  With ``gate_norm`` the log-gate is added; with ``dout``
    the gate gradient dg of Eq. 5 is returned too.
    """
    Hk = k.shape[1]
    Hq = q.shape[1]
    G = Hq // Hk
    kh = h // G
    n = k.shape[2]
    lo = u * q_block
    hi = min(n, lo + q_block)
    nc = sas_num_candidates(lo, b)
    s = np.asarray(scores[bi, h, u, :nc], dtype=np.float64)
    sel = topk_blocks(s, nc, K)
    gate = log_gates(s, nc, sel, gate_norm) if gate_norm else None
    kk, vv = k[bi, kh], v[bi, kh]
    o = np.zeros((hi - lo, q.shape[3]))
    lse = np.zeros(hi - lo)
    for t, i in enumerate(range(lo, hi)):
        o[t], lse[t] = sparse_attention_row(q[bi, h, i], kk, vv, i, b, sel, gate)
    res = {"idx": sel, "o": o, "lse": lse}
    if dout is not None and gate is not None:
        dg = gate_grad_rows(q[bi, h, lo:hi], kk, vv, range(lo, hi), b, sel, gate,
                            dout[bi, h, lo:hi])
        res["dg"] = np.array([dg[m] for m in sel])
    return res


def prefill_unit_reference_outer(q, k, v, scores, b, q_block, K, bi, h, u, gate_norm, dout=None):
    """prefill_unit_reference with the outer gate (R20): the same selection and softmax gate
    g_m = exp(log g_m), placed outside the softmax; dg of the outer gate with ``dout``."""
    Hk = k.shape[1]
    G = q.shape[1] // Hk
    kk, vv = k[bi, h // G], v[bi, h // G]
    n = k.shape[2]
    lo = u * q_block
    hi = min(n, lo + q_block)
    nc = sas_num_candidates(lo, b)
    s = np.asarray(scores[bi, h, u, :nc], dtype=np.float64)
    sel = topk_blocks(s, nc, K)
    g = {m: math.exp(lg) for m, lg in log_gates(s, nc, sel, gate_norm).items()}
    o = np.zeros((hi - lo, q.shape[3]))
    lse = np.zeros(hi - lo)
    for t, i in enumerate(range(lo, hi)):
        o[t], lse[t] = outer_gated_row(q[bi, h, i], kk, vv, i, b, sel, g)
    res = {"idx": sel, "o": o, "lse": lse}
    if dout is not None:
        dg = gate_grad_rows_outer(q[bi, h, lo:hi], kk, vv, range(lo, hi), b, sel,
                                  dout[bi, h, lo:hi])
        res["dg"] = np.array([dg[m] for m in sel])
    return res


# ----------------------------------------------------------------------------------------------
# FreeSolo two-branch prefill
# ----------------------------------------------------------------------------------------------


def rope(x, pos: int, theta: float = 10000.0):
    """Rotary position embedding of one vector at absolute position ``pos`` (R8).

    Rotate-half pairing: dimension t (t < d/2) pairs with t + d/2 and both rotate by the angle
    pos * theta^(-2t/d).  [FreeSolo] "How it works" applies RoPE inside the local window only.
    """
    x = np.asarray(x, dtype=np.float64)
    half = x.shape[0] // 2
    ang = pos * theta ** (-2.0 * np.arange(half) / x.shape[0])
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[:half], x[half:]
    return np.concatenate([a * c - b * s, b * c + a * s])


def freesolo_row(q, k, v, i, summaries, cell, q_block, K, window, lam, sigma, alpha, theta,
                 selection=None):
    """Two-branch output of the query at position i of one head ([FreeSolo] "How it works").

    Short branch: softmax attention of RoPE(q_i) over RoPE(k_j), j in [i-window+1, i].
    Long branch: candidate cells fixed by the query block, cell score r_ic, Top-K cells, one
    softmax over the raw (unrotated) tokens of those cells.  Mix (R8):
    o = (1 - alpha) o_short + alpha o_long; o = o_short when no cell is a candidate (R4).
    ``selection`` replaces the Top-K set by another set of candidate cells (used to evaluate the
    other valid sets of a near-tie).  Returns o, and the selected cells.
    """
    d = q.shape[0]
    mean_k, max_norm, centre = summaries
    lo = max(0, i - window + 1)
    qr = rope(q, i, theta)
    kr = np.array([rope(k[j], j, theta) for j in range(lo, i + 1)])
    z = kr @ qr / math.sqrt(d)
    w = np.exp(z - z.max())
    w /= w.sum()
    o_short = w @ np.asarray(v[lo:i + 1], dtype=np.float64)
    nc = freesolo_num_candidates(i, cell, q_block)
    if nc == 0 or (selection is not None and len(selection) == 0):
        return o_short, []
    r = round_f32(freesolo_scores(q, i, mean_k, max_norm, centre, lam, sigma, nc))
    sel = topk_blocks(r, nc, K) if selection is None else list(selection)
    toks = np.concatenate([np.arange(*block_range(c, k.shape[0], cell)) for c in sel])
    o_long, _, _ = attend(q, k, v, toks, np.zeros(len(toks)))
    return (1.0 - alpha) * o_short + alpha * o_long, sel


# ----------------------------------------------------------------------------------------------
# FS-B: forests of cell summaries searched by a beam (FreeSolo "How it differs")
# ----------------------------------------------------------------------------------------------


def fsb_high_cells(max_norm, n_cells: int) -> list[int]:
    """The cells of the second FS-B forest: those of norm at or above the median of the prefix.

    [FreeSolo] "How it differs" (FS-B): one forest holds the whole prefix, the other only the
    high-norm cells at or above the median.  R21: "at or above the median" is read as the
    ceil(n / 2) cells of largest maximum key norm (larger first, lower index on ties, NaN last) --
    the same set as norm >= median whenever no two norms tie at the middle, and always exactly
    half (rounded up).  Returns ascending cell indices.
    """
    return topk_blocks(max_norm, n_cells, (n_cells + 1) // 2)


def fsb_forest(cells, mean_k, max_norm, centre) -> list[dict]:
    """FS-B forest over ``cells`` (ascending): its nodes, each with the page's four summaries.

    [FreeSolo] "How it differs" (FS-B): every node stores a mean key, a radius, a maximum norm and
    a minimum position.  R21: the trees are perfect binary trees over consecutive cells in position
    order, one per set bit of the cell count, largest first (m = 13 cells give trees over the
    first 8, the next 4 and the last one); a node over leaves L has mean key mu = mean of their
    mean keys, radius rho = max over L of ||kbar_c - mu||_2, maximum norm = max over L of a_c and
    minimum position = min over L of p_c.  Returns every node as a dict with its leaves' range
    [lo, hi) in ``cells``, its height (leaves 0), whether it is a root, and the indices of its
    children in the returned list.
    """
    cells = [int(c) for c in cells]
    m = len(cells)
    nodes = []

    def build(lo, hi, height, root):
        leaves = cells[lo:hi]
        mu = np.mean([mean_k[c] for c in leaves], axis=0)
        rho = max(math.sqrt(float(np.dot(mean_k[c] - mu, mean_k[c] - mu))) for c in leaves)
        if height == 0:
            rho = 0.0
        node = {"lo": lo, "hi": hi, "height": height, "root": root, "first": leaves[0],
                "mu": mu, "rho": rho, "amax": max(float(max_norm[c]) for c in leaves),
                "pmin": min(float(centre[c]) for c in leaves), "children": []}
        at = len(nodes)
        nodes.append(node)
        if height > 0:
            mid = (lo + hi) // 2
            node["children"] = [build(lo, mid, height - 1, False),
                                build(mid, hi, height - 1, False)]
        return at

    lo = 0
    for h in range(max(m, 1).bit_length() - 1, -1, -1):
        if m & (1 << h):
            build(lo, lo + (1 << h), h, True)
            lo += 1 << h
    return nodes


def fsb_bound(node, q, i: int, lam: float, sigma: float) -> float:
    """Node score U_v: an upper bound of the cell score r_ic of every leaf below the node.

    [FreeSolo] "How it differs" (FS-B): U_v bounds the scores of the cells below v and justifies
    pruning.  R21: from the four summaries, q . kbar_c <= q . mu + ||q|| rho (Cauchy-Schwarz) and,
    with lambda >= 0 and the leaves in the query's past, a_c erf((i - p_c) / (2 sigma)) <=
    a_max erf((i - p_min) / (2 sigma)) (erf increasing, a_c <= a_max, p_c >= p_min):
        U_v = (q . mu + ||q|| rho) / sqrt(d) + lambda a_max erf((i - p_min) / (2 sigma)),
    which equals r_ic at a leaf (rho = 0).
    """
    q = np.asarray(q, dtype=np.float64)
    d = q.shape[0]
    dot = float(np.dot(q, node["mu"])) + math.sqrt(float(np.dot(q, q))) * node["rho"]
    return dot / math.sqrt(d) + lam * node["amax"] * float(_erf((i - node["pmin"]) / (2.0 * sigma)))


def fsb_beam(nodes, q, i: int, lam: float, sigma: float, width: int):
    """Beam search down one forest: the cells the beam reaches, and the smallest relative gap at
    any beam cut (how close the search came to a tie).

    [FreeSolo] "How it differs" (FS-B): a beam of W_b nodes per level descends the forest, ranked by
    U_v.  R21: level h holds the children of the previous level's beam and the roots of height h;
    the ``width`` best of them by U_v (rounded to float32, the decision precision; larger first,
    lower first cell on ties, NaN last) form the beam of level h; the beam of the leaf level is the
    set of candidate cells.
    """
    if not nodes:
        return [], math.inf
    top = max(n["height"] for n in nodes)
    beam = []
    gap = math.inf
    for h in range(top, -1, -1):
        pool = [c for b in beam for c in nodes[b]["children"]]
        pool += [j for j, n in enumerate(nodes) if n["root"] and n["height"] == h]
        scored = [(float(round_f32(fsb_bound(nodes[j], q, i, lam, sigma))), j) for j in pool]
        scored.sort(key=lambda x: _rank_key(x[0], nodes[x[1]]["first"]))
        if len(scored) > width:
            a, b = scored[width - 1][0], scored[width][0]
            if not (math.isnan(a) or math.isnan(b)):
                gap = min(gap, (a - b) / max(abs(a), abs(b), 1e-30))
        beam = [j for _, j in scored[:width]]
    return sorted(nodes[j]["first"] for j in beam), gap


def fsb_rerank_scores(q, k, cells, cell: int) -> np.ndarray:
    """Re-rank score of each candidate cell: log-sum-exp over the cell's tokens of the raw
    (unrotated) logits q . k_j / sqrt(d) ([FreeSolo] "How it differs", FS-B: the reached cells are
    re-ranked by logsumexp with their token keys)."""
    q = np.asarray(q, dtype=np.float64)
    d = q.shape[0]
    out = []
    for c in cells:
        lo, hi = block_range(int(c), k.shape[0], cell)
        z = np.asarray(k[lo:hi], dtype=np.float64) @ q / math.sqrt(d)
        out.append(logsumexp(z))
    return np.array(out)


def fsb_select(q, i: int, k, summaries, cell: int, q_block: int, K: int, lam: float,
               sigma: float, width: int):
    """FS-B selection of the query at position i: both forests over its candidate cells, a beam of
    ``width`` per level in each, the union of the cells reached, re-ranked by log-sum-exp over
    their tokens, top K (larger first, lower index on ties, NaN last; R11: the re-rank score is
    rounded to float32 before the decision).  Returns (selected cells ascending, candidate cells,
    smallest relative gap at a beam cut or at the final top-K cut)."""
    mean_k, max_norm, centre = summaries
    nc = freesolo_num_candidates(i, cell, q_block)
    if nc == 0:
        return [], [], math.inf
    cand = set()
    gap = math.inf
    for cells in (list(range(nc)), fsb_high_cells(max_norm, nc)):
        reached, g = fsb_beam(fsb_forest(cells, mean_k, max_norm, centre), q, i, lam, sigma, width)
        cand |= set(reached)
        gap = min(gap, g)
    cand = sorted(cand)
    r = round_f32(fsb_rerank_scores(q, k, cand, cell))
    order = sorted(range(len(cand)), key=lambda j: _rank_key(float(r[j]), cand[j]))
    if len(cand) > K:
        a, b = float(r[order[K - 1]]), float(r[order[K]])
        gap = min(gap, (a - b) / max(abs(a), abs(b), 1e-30))
    return sorted(cand[j] for j in order[:K]), cand, gap


# ----------------------------------------------------------------------------------------------
# Helpers the tests use to judge near-tie selections
# ----------------------------------------------------------------------------------------------


def selection_gap(s, n_cand: int, K: int):
    """(s_(K), s_(K+1)) of the descending order of the candidates, or None if n_cand <= K."""
    if n_cand <= K:
        return None
    order = sorted(range(n_cand), key=lambda c: _rank_key(float(s[c]), c))
    return float(s[order[K - 1]]), float(s[order[K]])


def valid_selections(s, n_cand: int, K: int, rel: float = 1e-4, limit: int = 64):
    """Every block set a selector may return for scores ``s`` (tie tolerance ``rel``).

    When the K-th and (K+1)-th largest scores differ by more than ``rel`` relative, only the exact
    Top-K set is valid.  Otherwise, with tau = rel * max(|s_(K)|, |s_(K+1)|), a valid set holds
    every block scoring above s_(K) + tau, K blocks in all, the rest drawn from the blocks within
    tau of s_(K).  Returns a list of ascending index lists, or None if there are more than
    ``limit`` of them.
    """
    s = np.asarray(s, dtype=np.float64)
    exact = topk_blocks(s, n_cand, K)
    gap = selection_gap(s, n_cand, K)
    if gap is None:
        return [exact]
    hi_s, lo_s = gap
    if math.isnan(hi_s) or math.isnan(lo_s):
        return [exact]
    tau = rel * max(abs(hi_s), abs(lo_s))
    if hi_s - lo_s > tau:
        return [exact]
    sure = [c for c in range(n_cand) if s[c] > hi_s + tau]
    maybe = [c for c in range(n_cand) if hi_s - tau <= s[c] <= hi_s + tau]
    need = K - len(sure)
    combos = list(itertools.islice(itertools.combinations(maybe, need), limit + 1))
    if len(combos) > limit:
        return None
    return [sorted(sure + list(cb)) for cb in combos]
