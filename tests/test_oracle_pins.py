"""Pins of the fp64 oracle against what the pages and the mathematics fix (CPU only).

Each test ties one oracle function to something other than itself: a value printed on a page, a
library routine the definition reduces to (torch's fp64 scaled-dot-product attention, NumPy
reductions), a closed form, an invariant, brute force, or finite differences.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import bsa_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def sdpa_causal(q, k, v):
    """Library reference: torch fp64 scaled_dot_product_attention with the causal mask."""
    q = torch.as_tensor(np.asarray(q, np.float64))[None, None]
    k = torch.as_tensor(np.asarray(k, np.float64))[None, None]
    v = torch.as_tensor(np.asarray(v, np.float64))[None, None]
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True)[0, 0].numpy()


def sdpa_full(q, k, v):
    q = torch.as_tensor(np.asarray(q, np.float64))[None, None]
    k = torch.as_tensor(np.asarray(k, np.float64))[None, None]
    v = torch.as_tensor(np.asarray(v, np.float64))[None, None]
    return torch.nn.functional.scaled_dot_product_attention(q, k, v)[0, 0].numpy()


def rnd(seed, *shape):
    return np.random.default_rng(seed).standard_normal(shape)


# ------------------------------------------------------------------------------------------
# Worked example printed on the SAS review page
# ------------------------------------------------------------------------------------------


def test_worked_example_gates_and_selection():
    ex = json.load(open(os.path.join(GOLDEN, "sas_worked_example.json")))
    s = np.array(ex["s"])
    C, K = ex["C"], ex["K"]
    assert orc.num_blocks(ex["n"], ex["b"]) == C
    # the query of the example sits in the block after the four history blocks
    i = C * ex["b"]
    assert orc.sas_num_candidates(i, ex["b"]) == C
    sel = orc.topk_blocks(s, C, K)
    assert sorted(m + 1 for m in sel) == sorted(ex["topk_one_based_printed"])
    lg = orc.log_gates(s, C, list(range(C)), "all")
    for m in range(C):
        assert abs(lg[m] - ex["log_g_printed"][m]) <= 0.025
    g = {m: math.exp(lg[m]) for m in range(C)}
    assert abs(sum(g.values()) - 1.0) < 1e-15  # softmax gates sum to one
    for m in range(C):
        assert abs(math.exp(s[m]) - ex["exp_s_printed"][m]) <= 0.006
    assert abs(sum(math.exp(x) for x in s) - ex["sum_exp_printed"]) <= 0.006
    # biases injected on the selected blocks (step 4): B_2 gets ~-0.80, B_1 ~-1.47
    lg_sel = orc.log_gates(s, C, sel, "all")
    assert abs(lg_sel[1] - ex["bias_on_B2_printed"]) <= 0.025
    assert abs(lg_sel[0] - ex["bias_on_B1_printed"]) <= 0.025
    # the gate of the top block is the largest: block 2 (1-based) is the most important
    assert max(lg, key=lg.get) == 1


def test_worked_example_gate_enters_inside_softmax():
    """Step 4: with the gate inside the softmax, B_2 receives more mass than B_1 for equal logits."""
    ex = json.load(open(os.path.join(GOLDEN, "sas_worked_example.json")))
    b, C, K = ex["b"], ex["C"], ex["K"]
    d = 8
    n = C * b + 1  # one token of the current block
    k = np.zeros((n, d))  # equal logits everywhere
    v = np.zeros((n, d))
    v[0 * b:1 * b, 0] = 1.0  # B_1 marks dimension 0
    v[1 * b:2 * b, 1] = 1.0  # B_2 marks dimension 1
    s = np.array(ex["s"])
    sel = orc.topk_blocks(s, C, K)
    gate = orc.log_gates(s, C, sel, "all")
    o, _ = orc.sparse_attention_row(np.ones(d), k, v, n - 1, b, sel, gate)
    assert o[1] > o[0] > 0
    # mass ratio equals the gate ratio exp(-0.79)/exp(-1.49) = exp(0.7)
    assert abs(o[1] / o[0] - math.exp(s[1] - s[0])) < 1e-12


# ------------------------------------------------------------------------------------------
# Exact sparse softmax = dense attention in the special cases the definition reduces to
# ------------------------------------------------------------------------------------------


@pytest.mark.parametrize("n,b", [(200, 64), (256, 64), (67, 16)])
def test_all_blocks_equals_dense_causal(n, b):
    d = 16
    q, k, v = rnd(1, n, d), rnd(2, n, d), rnd(3, n, d)
    ref = sdpa_causal(q, k, v)
    for i in range(n):
        nc = orc.sas_num_candidates(i, b)
        sel = orc.topk_blocks(rnd(4 + i, nc), nc, K=10**6)
        assert sel == list(range(nc))
        o, _ = orc.sparse_attention_row(q[i], k, v, i, b, sel)
        assert np.max(np.abs(o - ref[i])) < 1e-12


def test_gqa_decode_all_blocks_equals_dense():
    B, Hq, Hk, d, n, b = 2, 4, 2, 8, 150, 32
    q = rnd(5, B, Hq, d)
    k, v = rnd(6, B, Hk, n, d), rnd(7, B, Hk, n, d)
    seq = np.array([150, 97], dtype=np.int32)
    res = orc.decode_reference(q, k, v, seq, b, K=100)
    for bi in range(B):
        L = seq[bi]
        qt = torch.as_tensor(q[bi][:, None, :])  # [Hq, 1, d]
        kt = torch.as_tensor(k[bi, :, :L])
        vt = torch.as_tensor(v[bi, :, :L])
        ref = torch.nn.functional.scaled_dot_product_attention(qt[None], kt[None], vt[None],
                                                               enable_gqa=True)[0, :, 0].numpy()
        for h in range(Hq):
            assert np.max(np.abs(res[(bi, h)]["o"] - ref[h])) < 1e-12
            # lse pinned by its definition through the same library logits
            z = (kt[h // (Hq // Hk)] @ qt[h, 0]).numpy() / math.sqrt(d)
            assert abs(res[(bi, h)]["lse"] - float(torch.logsumexp(torch.as_tensor(z), 0))) < 1e-12


def test_gather_equals_dense_mask_with_gate():
    """The gather path equals an independently built dense-mask computation (Monodratic)."""
    n, b, d = 300, 32, 12
    q, k, v = rnd(8, n, d), rnd(9, n, d), rnd(10, n, d)
    rng = np.random.default_rng(11)
    for i in [0, 31, 32, 100, 255, 299]:
        nc = orc.sas_num_candidates(i, b)
        s = rng.standard_normal(nc)
        sel = orc.topk_blocks(s, nc, 3)
        for norm in [None, "selected", "all"]:
            gate = orc.log_gates(s, nc, sel, norm) if norm else None
            o1, _ = orc.sparse_attention_row(q[i], k, v, i, b, sel, gate)
            o2 = orc.masked_attention_row(q[i], k, v, i, b, sel, gate)
            assert np.max(np.abs(o1 - o2)) < 1e-12


def test_weights_sum_to_one_and_causal():
    n, b, d = 130, 16, 8
    q, k, v = rnd(12, n, d), rnd(13, n, d), rnd(14, n, d)
    for i in [0, 15, 16, 77, 129]:
        nc = orc.sas_num_candidates(i, b)
        sel = orc.topk_blocks(rnd(15 + i, nc), nc, 2)
        toks, owner = orc.token_set(i, b, sel, n)
        assert toks.max() <= i  # no token after the query
        assert all(m < i // b for m in sel)  # no selected block in the future
        assert set(toks[owner == -1]) == set(range((i // b) * b, i + 1))  # current block kept
        _, _, p = orc.attend(q[i], k, v, toks, np.zeros(len(toks)))
        assert abs(p.sum() - 1.0) < 1e-14 and (p >= 0).all()


def test_explicit_causal_mask_equals_implicit():
    """Mask plumbing check (attention-sink post): an explicit causal mask equals is_causal."""
    n, d = 40, 8
    q, k, v = rnd(16, n, d), rnd(17, n, d), rnd(18, n, d)
    ref = sdpa_causal(q, k, v)
    for i in range(n):
        o = orc.masked_attention_row(q[i], k, v, i, b=8, selected=range(i // 8))
        assert np.max(np.abs(o - ref[i])) == pytest.approx(0.0, abs=1e-13)


# ------------------------------------------------------------------------------------------
# Top-K against brute force
# ------------------------------------------------------------------------------------------


def brute_topk(s, n_cand, K):
    """The unique K-subset whose every member outranks every non-member."""
    def beats(a, bb):
        xa, xb = s[a], s[bb]
        if math.isnan(xa):
            return math.isnan(xb) and a < bb
        if math.isnan(xb):
            return True
        return xa > xb or (xa == xb and a < bb)
    kk = min(K, n_cand)
    found = []
    for sub in itertools.combinations(range(n_cand), kk):
        rest = [c for c in range(n_cand) if c not in sub]
        if all(beats(a, r) for a in sub for r in rest):
            found.append(list(sub))
    assert len(found) == 1
    return found[0]


def test_topk_bruteforce_exhaustive_small_alphabet():
    alphabet = [-1.0, 0.0, 0.5, 2.0, float("nan"), -math.inf]
    for C in range(1, 5):
        for vals in itertools.product(alphabet, repeat=C):
            s = np.array(vals)
            for K in range(1, C + 1):
                for nc in range(0, C + 1):
                    assert orc.topk_blocks(s, nc, K) == brute_topk(s, nc, K)


def test_topk_bruteforce_random_with_ties():
    rng = np.random.default_rng(19)
    for _ in range(300):
        C = int(rng.integers(1, 9))
        s = rng.integers(-2, 3, size=C).astype(np.float64)  # heavy ties
        K = int(rng.integers(1, C + 1))
        nc = int(rng.integers(0, C + 1))
        assert orc.topk_blocks(s, nc, K) == brute_topk(s, nc, K)


def test_topk_signed_zero_ties_by_index():
    s = np.array([0.0, -0.0, 0.0, -0.0])
    assert orc.topk_blocks(s, 4, 2) == [0, 1]


def test_valid_selections_near_tie():
    s = np.array([1.0, 0.99999999, 0.5, 1.0000000001])
    sets = orc.valid_selections(s, 4, 2)
    assert [0, 3] in sets and [1, 3] in sets and len(sets) >= 2
    assert orc.valid_selections(np.array([3.0, 1.0, 2.0]), 3, 2) == [[0, 2]]


# ------------------------------------------------------------------------------------------
# Gate
# ------------------------------------------------------------------------------------------


def test_uniform_scores_give_constant_bias():
    for nc, K in [(10, 3), (5, 5), (7, 1)]:
        s = np.full(nc, 0.37)
        sel = orc.topk_blocks(s, nc, K)
        assert sel == list(range(K))  # ties: lowest indices
        lg_sel = orc.log_gates(s, nc, sel, "selected")
        lg_all = orc.log_gates(s, nc, sel, "all")
        for m in sel:
            assert abs(lg_sel[m] + math.log(K)) < 1e-14
            assert abs(lg_all[m] + math.log(nc)) < 1e-14


def test_single_selected_block_gate_is_one():
    n, b, d = 200, 32, 8
    q, k, v = rnd(20, n, d), rnd(21, n, d), rnd(22, n, d)
    i = 150
    nc = orc.sas_num_candidates(i, b)
    s = rnd(23, nc)
    sel = orc.topk_blocks(s, nc, 1)
    gate = orc.log_gates(s, nc, sel, "selected")
    assert abs(gate[sel[0]]) < 1e-15
    o1, l1 = orc.sparse_attention_row(q[i], k, v, i, b, sel, gate)
    o0, l0 = orc.sparse_attention_row(q[i], k, v, i, b, sel)
    assert np.max(np.abs(o1 - o0)) < 1e-15 and abs(l1 - l0) < 1e-13


def test_uniform_gate_over_selected_is_rescaled_history():
    """A constant bias -log K moves mass from history to the current block by exactly K."""
    n, b, d = 160, 32, 4
    q = np.zeros(d)
    k = np.zeros((n, d))
    v = np.zeros((n, d))
    i = 140
    nc = orc.sas_num_candidates(i, b)
    sel = [0, 2]
    v[0:32, 0] = 1
    v[64:96, 0] = 1
    gate = orc.log_gates(np.zeros(nc), nc, sel, "selected")
    o, _ = orc.sparse_attention_row(q, k, v, i, b, sel, gate)
    n_hist, n_cur = 64, i - 128 + 1
    assert abs(o[0] - (n_hist / 2) / (n_hist / 2 + n_cur)) < 1e-14


def test_gate_gradient_matches_finite_differences():
    n, b, d = 256, 32, 8
    rng = np.random.default_rng(24)
    q, k, v = rng.standard_normal((n, d)), rng.standard_normal((n, d)), rng.standard_normal((n, d))
    do = rng.standard_normal((n, d))
    lo, hi = 192, 224  # one unit of 32 queries
    nc = orc.sas_num_candidates(lo, b)
    s = rng.standard_normal(nc)
    sel = orc.topk_blocks(s, nc, 3)
    for norm in ["selected", "all"]:
        gate = orc.log_gates(s, nc, sel, norm)
        g = {m: math.exp(gate[m]) for m in sel}
        pos = list(range(lo, hi))
        dg = orc.gate_grad_rows(q[lo:hi], k, v, pos, b, sel, gate, do[lo:hi])
        for m in sel:
            h = 1e-6 * g[m]
            gp, gm = dict(g), dict(g)
            gp[m] += h
            gm[m] -= h
            fd = (orc.gated_loss(q[lo:hi], k, v, pos, b, sel, gp, do[lo:hi]) -
                  orc.gated_loss(q[lo:hi], k, v, pos, b, sel, gm, do[lo:hi])) / (2 * h)
            assert abs(dg[m] - fd) <= 1e-6 * max(1.0, abs(fd))


def _loss_of_scores(s, nc, sel, norm, q, k, v, pos, b, do):
    gate = orc.log_gates(s, nc, sel, norm)
    g = {m: math.exp(gate[m]) for m in sel}
    return orc.gated_loss(q, k, v, pos, b, sel, g, do)


def test_selector_gradient_matches_finite_differences():
    """ds through the log-softmax gate equals central differences of the gated loss in every
    history score -- the unselected ones included when the normaliser runs over all history."""
    n, b, d = 256, 32, 8
    rng = np.random.default_rng(29)
    q, k, v = rng.standard_normal((n, d)), rng.standard_normal((n, d)), rng.standard_normal((n, d))
    do = rng.standard_normal((n, d))
    lo, hi = 192, 224
    nc = orc.sas_num_candidates(lo, b)
    s = rng.standard_normal(nc)
    sel = orc.topk_blocks(s, nc, 3)
    pos = list(range(lo, hi))
    for norm in ["selected", "all"]:
        gate = orc.log_gates(s, nc, sel, norm)
        dg = orc.gate_grad_rows(q[lo:hi], k, v, pos, b, sel, gate, do[lo:hi])
        ds = orc.selector_grad_row(s, nc, sel, dg, norm)
        for c in range(nc):
            h = 1e-6
            sp, sm = s.copy(), s.copy()
            sp[c] += h
            sm[c] -= h
            fd = (_loss_of_scores(sp, nc, sel, norm, q[lo:hi], k, v, pos, b, do[lo:hi]) -
                  _loss_of_scores(sm, nc, sel, norm, q[lo:hi], k, v, pos, b, do[lo:hi])) / (2 * h)
            assert abs(ds[c] - fd) <= 1e-6 * max(1.0, abs(fd)), (norm, c, ds[c], fd)
        if norm == "selected":
            assert all(ds[c] == 0.0 for c in range(nc) if c not in sel)


def test_selector_gradient_sums_to_zero():
    """Adding one constant to every score of the normaliser set leaves the gates unchanged, so
    the gradient sums to zero over that set."""
    rng = np.random.default_rng(30)
    nc, K = 40, 6
    s = rng.standard_normal(nc)
    sel = orc.topk_blocks(s, nc, K)
    dg = {m: float(rng.standard_normal()) for m in sel}
    ds_all = orc.selector_grad_row(s, nc, sel, dg, "all")
    ds_sel = orc.selector_grad_row(s, nc, sel, dg, "selected")
    assert abs(ds_all.sum()) < 1e-12 * max(1.0, np.abs(ds_all).max() * nc)
    assert abs(ds_sel.sum()) < 1e-12 * max(1.0, np.abs(ds_sel).max() * nc)
    # a planted sign error in the normaliser term breaks the invariant
    g = {m: math.exp(v) for m, v in orc.log_gates(s, nc, sel, "all").items()}
    wrong = ds_all.copy()
    for m in sel:
        wrong[m] += 2 * g[m] * dg[m]
    assert abs(wrong.sum()) > 1e-6


def test_prefill_unit_dg_matches_rows():
    """The unit driver sums Eq. 5 over the unit's queries (R10) and picks Top-K of its scores."""
    B, Hq, Hk, n, d, b, qb, K = 1, 2, 1, 256, 8, 32, 32, 2
    rng = np.random.default_rng(25)
    q, k, v = rng.standard_normal((B, Hq, n, d)), rng.standard_normal((B, Hk, n, d)), \
        rng.standard_normal((B, Hk, n, d))
    do = rng.standard_normal((B, Hq, n, d))
    s = rng.standard_normal((B, Hq, n // qb, n // b))
    res = orc.prefill_unit_reference(q, k, v, s, b, qb, K, 0, 1, 5, "selected", do)
    nc = 5
    sel = orc.topk_blocks(s[0, 1, 5], nc, K)
    assert res["idx"] == sel
    gate = orc.log_gates(s[0, 1, 5], nc, sel, "selected")
    rows = range(160, 192)
    dg = orc.gate_grad_rows(q[0, 1, 160:192], k[0, 0], v[0, 0], rows, b, sel, gate, do[0, 1, 160:192])
    assert np.allclose(res["dg"], [dg[m] for m in sel], rtol=0, atol=1e-14)


# ------------------------------------------------------------------------------------------
# Summaries
# ------------------------------------------------------------------------------------------


def test_summaries_closed_forms():
    d, b = 6, 16
    kv = rnd(26, d)
    k = np.tile(kv, (40, 1))  # constant keys, ragged final block of 8
    mean_k, max_norm, centre = orc.block_summaries(k, b)
    assert mean_k.shape == (3, d)
    assert np.max(np.abs(mean_k - kv)) < 1e-15
    assert np.max(np.abs(max_norm - np.linalg.norm(kv))) < 1e-14
    assert list(centre) == [7.5, 23.5, 35.5]  # c*b + (b-1)/2, ragged block: 32 + 7/2


def test_summaries_against_numpy_reductions():
    k = rnd(27, 100, 5)
    mean_k, max_norm, _ = orc.block_summaries(k, 32)
    for c, (lo, hi) in enumerate([(0, 32), (32, 64), (64, 96), (96, 100)]):
        assert np.allclose(mean_k[c], np.mean(k[lo:hi], axis=0), atol=1e-15, rtol=0)
        assert abs(max_norm[c] - np.max(np.linalg.norm(k[lo:hi], axis=1))) < 1e-14


def test_dot_scores_value():
    q = np.array([1.0, 2.0, 0.0, -1.0])
    mean_k = np.array([[0.5, 0.5, 3.0, 1.0], [1.0, 0.0, 0.0, 0.0]])
    assert np.allclose(orc.dot_scores(q, mean_k, 2), [0.25, 0.5], atol=1e-15)


# ------------------------------------------------------------------------------------------
# FreeSolo
# ------------------------------------------------------------------------------------------


def test_freesolo_score_value_and_sign():
    q = np.array([2.0, 0.0, 0.0, 0.0])
    mean_k = np.array([[1.0, 0.0, 0.0, 0.0], [1.0, 0.0, 0.0, 0.0]])
    max_norm = np.array([3.0, 3.0])
    centre = np.array([15.5, 47.5])
    i, lam, sigma = 47.5 + 2 * 40.0 * 0.5, 0.5, 40.0  # (i - p_1)/(2 sigma) = 0.5
    r = orc.freesolo_scores(q, i, mean_k, max_norm, centre, lam, sigma, 2)
    assert abs(r[1] - (1.0 + 0.5 * 3.0 * math.erf(0.5))) < 1e-14
    assert r[0] > r[1]  # the farther past cell gets the larger positive bias
    assert np.allclose(orc.freesolo_scores(q, i, mean_k, max_norm, centre, 0.0, sigma, 2),
                       orc.dot_scores(q, mean_k, 2), atol=0)


def test_freesolo_candidates_fixed_per_query_block():
    for i in range(0, 1024, 7):
        nc = orc.freesolo_num_candidates(i, 32, 128)
        assert nc * 32 <= (i // 128) * 128 <= i
        assert nc == orc.freesolo_num_candidates((i // 128) * 128, 32, 128)


def test_rope_properties():
    d = 16
    x, y = rnd(28, d), rnd(29, d)
    for p in [0, 1, 17, 1000]:
        assert abs(np.linalg.norm(orc.rope(x, p)) - np.linalg.norm(x)) < 1e-12
    # relative-position invariance of the rotated dot product
    for i, j, t in [(5, 3, 11), (100, 0, 7), (40, 39, 1000)]:
        a = np.dot(orc.rope(x, i), orc.rope(y, j))
        bb = np.dot(orc.rope(x, i + t), orc.rope(y, j + t))
        assert abs(a - bb) < 1e-10
    # d = 2: a plane rotation by angle pos (the first frequency is theta^0 = 1)
    z = orc.rope(np.array([1.0, 0.0]), 3)
    assert np.allclose(z, [math.cos(3), math.sin(3)], atol=1e-15)
    assert np.allclose(orc.rope(x, 0), x, atol=0)


def test_rope_hand_values():
    """R8 written out by hand for d = 4 at position 100 (base 10000, rotate-half pairing): the
    pair (0, 2) turns by 100 * 10000^0 = 100 rad and the pair (1, 3) by 100 * 10000^(-2/4) = 1 rad.
    cos 100 = 0.8623188722876839, sin 100 = -0.5063656411097588 (100 - 15 * 2 pi = 5.7522 rad),
    cos 1 = 0.5403023058681398, sin 1 = 0.8414709848078965.  An interleaved pairing ((0, 1),
    (2, 3)) or another frequency exponent (for example 10000^(-t/d)) gives other numbers."""
    got = orc.rope(np.array([1.0, 2.0, 3.0, 4.0]), 100)
    want = [1 * 0.8623188722876839 - 3 * -0.5063656411097588,   # 2.3814157956169604
            2 * 0.5403023058681398 - 4 * 0.8414709848078965,    # -2.2852793274953065
            3 * 0.8623188722876839 + 1 * -0.5063656411097588,   # 2.0805909757532928
            4 * 0.5403023058681398 + 2 * 0.8414709848078965]    # 3.844151193088352
    assert np.allclose(got, want, rtol=0, atol=1e-13)
    assert np.allclose(got, [2.3814157956169604, -2.2852793274953065, 2.0805909757532928,
                             3.844151193088352], rtol=0, atol=1e-13)
    # the same rotation as complex multiplication: (x_t + i x_{t+d/2}) * exp(i pos theta^(-2t/d))
    d, pos = 8, 37
    x = rnd(33, d)
    z = (x[:d // 2] + 1j * x[d // 2:]) * np.exp(1j * pos * 10000.0 ** (-np.arange(d // 2) / (d / 2)))
    assert np.allclose(orc.rope(x, pos), np.concatenate([z.real, z.imag]), atol=1e-13)


def test_freesolo_infinite_window_short_branch_is_dense_rope_attention():
    n, d, cell, qb = 96, 8, 8, 32
    q, k, v = rnd(30, n, d), rnd(31, n, d), rnd(32, n, d)
    summ = orc.block_summaries(k, cell)
    qr = np.array([orc.rope(q[i], i) for i in range(n)])
    kr = np.array([orc.rope(k[j], j) for j in range(n)])
    ref = sdpa_causal(qr, kr, v)
    for i in [0, 5, 31, 32, 64, 95]:
        o, _ = orc.freesolo_row(q[i], k, v, i, summ, cell, qb, 2, window=10**6, lam=0.5,
                                sigma=100.0, alpha=0.0, theta=10000.0)
        assert np.max(np.abs(o - ref[i])) < 1e-12


def test_freesolo_long_branch_all_cells_is_prefix_attention():
    n, d, cell, qb = 96, 8, 8, 32
    q, k, v = rnd(33, n, d), rnd(34, n, d), rnd(35, n, d)
    summ = orc.block_summaries(k, cell)
    for i in [32, 50, 64, 95]:
        prefix = (i // qb) * qb
        o, sel = orc.freesolo_row(q[i], k, v, i, summ, cell, qb, K=100, window=4, lam=0.5,
                                  sigma=100.0, alpha=1.0, theta=10000.0)
        assert sel == list(range(prefix // cell))
        ref = sdpa_full(q[i:i + 1], k[:prefix], v[:prefix])[0]  # NoPE over the prefix
        assert np.max(np.abs(o - ref)) < 1e-12


def test_freesolo_mix_and_first_query_block():
    n, d, cell, qb = 64, 4, 8, 32
    q, k, v = rnd(36, n, d), rnd(37, n, d), rnd(38, n, d)
    summ = orc.block_summaries(k, cell)
    args = dict(cell=cell, q_block=qb, K=2, window=16, lam=0.5, sigma=50.0, theta=10000.0)
    o0, sel0 = orc.freesolo_row(q[10], k, v, 10, summ, alpha=0.7, **args)
    os_, _ = orc.freesolo_row(q[10], k, v, 10, summ, alpha=0.0, **args)
    assert sel0 == [] and np.max(np.abs(o0 - os_)) < 1e-15  # no candidate: short branch alone
    i = 50
    o_s, _ = orc.freesolo_row(q[i], k, v, i, summ, alpha=0.0, **args)
    o_l, _ = orc.freesolo_row(q[i], k, v, i, summ, alpha=1.0, **args)
    o_m, _ = orc.freesolo_row(q[i], k, v, i, summ, alpha=0.25, **args)
    assert np.max(np.abs(o_m - (0.75 * o_s + 0.25 * o_l))) < 1e-14


# ------------------------------------------------------------------------------------------
# Planted mistakes: the pins above catch a wrong oracle (mistakes planted on the CPU only)
# ------------------------------------------------------------------------------------------


def test_planted_mistakes_are_caught(monkeypatch):
    n, b, d = 64, 16, 8
    q, k, v = rnd(39, n, d), rnd(40, n, d), rnd(41, n, d)
    ref = sdpa_causal(q, k, v)

    def worst():
        err = 0.0
        for i in range(n):
            nc = orc.sas_num_candidates(i, b)
            o, _ = orc.sparse_attention_row(q[i], k, v, i, b, list(range(nc)))
            err = max(err, float(np.max(np.abs(o - ref[i]))))
        return err

    assert worst() < 1e-12
    good_attend = orc.attend

    def attend_no_scale(qq, kk, vv, toks, bias):  # dropped 1/sqrt(d)
        return good_attend(qq * math.sqrt(len(qq)), kk, vv, toks, bias)

    monkeypatch.setattr(orc, "attend", attend_no_scale)
    assert worst() > 1e-3
    monkeypatch.setattr(orc, "attend", good_attend)

    good_range = orc.block_range
    monkeypatch.setattr(orc, "block_range", lambda c, nn, bb: (c * bb, min(nn, (c + 1) * bb - 1)))
    assert worst() > 1e-3  # a block that loses its last token
    monkeypatch.setattr(orc, "block_range", good_range)


def test_freesolo_explicit_selection_matches_default():
    n, d, cell, qb = 96, 8, 8, 32
    q, k, v = rnd(42, n, d), rnd(43, n, d), rnd(44, n, d)
    summ = orc.block_summaries(k, cell)
    args = dict(cell=cell, q_block=qb, K=2, window=16, lam=0.5, sigma=50.0, alpha=0.4,
                theta=10000.0)
    for i in [40, 70, 95]:
        o1, sel = orc.freesolo_row(q[i], k, v, i, summ, **args)
        o2, sel2 = orc.freesolo_row(q[i], k, v, i, summ, selection=sel, **args)
        assert sel2 == sel and np.max(np.abs(o1 - o2)) == 0.0
        o3, _ = orc.freesolo_row(q[i], k, v, i, summ, selection=[0], **args)
        assert np.max(np.abs(o3 - o1)) > 0  # a different set changes the long branch


def test_fsl_candidates_against_brute_force():
    """FS-L pruning = the W newest cells plus, among the older ones, the P largest norms (lower
    index on ties, NaN last), checked against a direct sort; small and degenerate sizes."""
    rng = np.random.default_rng(40)
    for trial in range(200):
        n_cells = int(rng.integers(0, 40))
        W, P = int(rng.integers(0, 6)), int(rng.integers(0, 10))
        a = np.round(rng.standard_normal(n_cells) * 2) / 2  # many ties
        if n_cells > 3 and trial % 7 == 0:
            a[1] = np.nan
        got = orc.fsl_candidates(a, n_cells, W, P)
        recent = set(range(max(0, n_cells - W), n_cells))
        older = [c for c in range(n_cells) if c not in recent]
        keyed = sorted(older, key=lambda c: (1, 0.0, c) if np.isnan(a[c]) else (0, -a[c], c))
        want = sorted(recent | set(keyed[:P]))
        assert got == want
        assert len(got) == min(n_cells, W + P)
        # properties, independent of how the set is built: the recent cells are kept, and every
        # kept older cell outranks every dropped older cell
        assert recent <= set(got)
        kept_old = [c for c in got if c not in recent]
        dropped = [c for c in older if c not in got]

        def outranks(x, y):
            if np.isnan(a[y]):
                return not np.isnan(a[x]) or x < y
            if np.isnan(a[x]):
                return False
            return a[x] > a[y] or (a[x] == a[y] and x < y)
        assert all(outranks(x, y) for x in kept_old for y in dropped)


def test_fsl_select_with_every_cell_kept_is_the_full_selection():
    """When the pruned set holds every cell, FS-L selection equals the full method's Top-K."""
    rng = np.random.default_rng(41)
    n, d, cell = 2048, 16, 32
    k = rng.standard_normal((n, d))
    mean_k, max_norm, centre = orc.block_summaries(k, cell)
    for i in [300, 1000, 2047]:
        q = rng.standard_normal(d)
        nc = orc.freesolo_num_candidates(i, cell, 128)
        cand = orc.fsl_candidates(max_norm, nc, W=8, P=nc)
        assert cand == list(range(nc))
        full = orc.topk_blocks(orc.round_f32(orc.freesolo_scores(q, i, mean_k, max_norm, centre,
                                                                 0.5, 300.0, nc)), nc, 4)
        assert orc.fsl_select(q, i, mean_k, max_norm, centre, 0.5, 300.0, cand, 4) == full
    # a pruned set: the selection stays inside it
    cand = orc.fsl_candidates(max_norm, 40, W=8, P=5)
    got = orc.fsl_select(rng.standard_normal(d), 1400, mean_k, max_norm, centre, 0.5, 300.0,
                         cand, 4)
    assert set(got) <= set(cand) and len(got) == 4


def test_fsl_state_update_equals_the_pruning_recomputed_from_scratch():
    """The O(W + P) state update (one cell at a time, the cell leaving the W newest competing with
    the lowest-ranked kept older cell) keeps exactly the set the pruning rule picks from the whole
    prefix, after every growth step; ties and NaN norms included."""
    rng = np.random.default_rng(42)
    for trial in range(120):
        total = int(rng.integers(1, 120))
        W, P = int(rng.integers(0, 9)), int(rng.integers(0, 12))
        a = np.round(rng.standard_normal(total) * 2) / 2  # many ties
        if trial % 5 == 0:
            a[rng.integers(0, total, 3)] = np.nan
        st = orc.fsl_state_new(W, P)
        n = 0
        while n < total:
            n = min(total, n + int(rng.integers(0, 6)))
            st = orc.fsl_state_advance(st, a, n)
            assert orc.fsl_state_cells(st) == orc.fsl_candidates(a, n, W, P), (trial, n)
            assert len(st["older"]) <= P
    # the state never looks past its P cells: a norm changed after a cell was dropped does not
    # bring it back (the update reads only the joining cell and the kept ones)
    a = np.array([5.0, 1.0, 4.0, 0.5, 0.2, 0.1])
    st = orc.fsl_state_advance(orc.fsl_state_new(1, 2), a, 6)
    assert orc.fsl_state_cells(st) == [0, 2, 5]


def test_fsl_decode_row_keeping_every_cell_is_the_full_method():
    """With W + P covering every candidate cell the FS-L decode output equals the full method's
    two-branch output; with a pruned state its long branch reads only kept cells."""
    rng = np.random.default_rng(43)
    n, d, cell = 1536, 16, 32
    q, k, v = rng.standard_normal((n, d)), rng.standard_normal((n, d)), rng.standard_normal((n, d))
    summ = orc.block_summaries(k, cell)
    for i in [200, 700, 1535]:
        nc = orc.freesolo_num_candidates(i, cell, 128)
        st = orc.fsl_state_advance(orc.fsl_state_new(8, nc), summ[1], nc)
        cand = orc.fsl_state_cells(st)
        o1, sel1 = orc.fsl_decode_row(q[i], k, v, i, summ, cand, cell, 4, 256, 0.5, 300.0, 0.3,
                                      10000.0)
        o2, sel2 = orc.freesolo_row(q[i], k, v, i, summ, cell, 128, 4, 256, 0.5, 300.0, 0.3,
                                    10000.0)
        assert sel1 == sel2
        assert np.allclose(o1, o2, atol=1e-12)
    i = 1535
    nc = orc.freesolo_num_candidates(i, cell, 128)
    st = orc.fsl_state_advance(orc.fsl_state_new(2, 3), summ[1], nc)
    cand = orc.fsl_state_cells(st)
    o, sel = orc.fsl_decode_row(q[i], k, v, i, summ, cand, cell, 4, 256, 0.5, 300.0, 0.3, 10000.0)
    assert set(sel) <= set(cand) and len(sel) == 4
    o_ref, _ = orc.freesolo_row(q[i], k, v, i, summ, cell, 128, 4, 256, 0.5, 300.0, 0.3, 10000.0,
                                selection=sel)
    assert np.allclose(o, o_ref, atol=1e-12)


# ------------------------------------------------------------------------------------------
# bf16 summaries and GQA-shared selection (R19)
# ------------------------------------------------------------------------------------------


def _bf16_by_grid(x: float) -> float:
    """bfloat16 rounding rebuilt from the number line: the grid spacing at |x| is 2^(e - 7) with
    e = max(floor(log2 |x|), -126); take the nearer grid neighbour, the even multiple on a tie."""
    if x == 0.0 or math.isinf(x):
        return x
    a = abs(x)
    e = max(math.floor(math.log2(a)), -126)
    ulp = 2.0 ** (e - 7)
    lo = math.floor(a / ulp)
    r = a / ulp - lo
    m = lo + 1 if (r > 0.5 or (r == 0.5 and lo % 2 == 1)) else lo
    return math.copysign(m * ulp, x)


def test_round_bf16_matches_grid_construction():
    rng = np.random.default_rng(90)
    x = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
        rng.standard_normal(2000) * 1e-39,            # float32 subnormals
    ]).astype(np.float32)
    got = orc.round_bf16(x)
    ref = np.array([_bf16_by_grid(float(v)) for v in x])
    assert np.array_equal(got, ref)


def test_round_bf16_ties_and_specials():
    # ties: exactly half a bf16 step above a grid point round to the even significand
    assert orc.round_bf16(1.0 + 2.0 ** -8) == 1.0             # 1.0000000|1 -> even 1.0
    assert orc.round_bf16(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6
    assert orc.round_bf16(-(1.0 + 2.0 ** -8)) == -1.0
    assert orc.round_bf16(1.0 + 2.0 ** -8 + 2.0 ** -20) == 1.0 + 2.0 ** -7  # just above half
    # representable values are kept; infinities stay; the largest float32 overflows to infinity
    for v in [0.0, -0.0, 1.5, -3.25, 2.0 ** -133, np.inf, -np.inf]:
        assert orc.round_bf16(v) == v
    assert orc.round_bf16(np.finfo(np.float32).max) == np.inf
    assert np.isnan(orc.round_bf16(np.nan))


def test_shared_scores_are_the_mean_query_scores():
    """Mean over heads of q_g . kbar / sqrt(d) equals the mean query's score (linearity)."""
    rng = np.random.default_rng(91)
    G, d, C = 4, 64, 40
    qs = rng.standard_normal((G, d))
    mean_k = rng.standard_normal((C, d))
    per_head = [orc.dot_scores(qs[g], mean_k, C) for g in range(G)]
    shared = orc.shared_block_scores(per_head)
    assert np.allclose(shared, orc.dot_scores(qs.mean(axis=0), mean_k, C), rtol=0, atol=1e-12)
    assert np.allclose(orc.shared_block_scores(per_head[::-1]), shared, rtol=0, atol=1e-14)


def test_shared_selection_reduces_to_per_head():
    """One query head per kv head: the shared decode step is the per-head decode step; identical
    heads in a group: every head keeps its own selection."""
    rng = np.random.default_rng(92)
    B, Hk, n, d, b, K = 2, 2, 700, 32, 32, 4
    k = rng.standard_normal((B, Hk, n, d))
    v = rng.standard_normal((B, Hk, n, d))
    seq = np.array([700, 333])
    q1 = rng.standard_normal((B, Hk, d))
    a = orc.decode_reference_shared(q1, k, v, seq, b, K)
    r = orc.decode_reference(q1, k, v, seq, b, K)
    for key in r:
        assert a[key]["idx"] == r[key]["idx"]
        assert np.allclose(a[key]["o"], r[key]["o"], rtol=0, atol=1e-12)
    q4 = np.repeat(q1, 4, axis=1)   # four identical heads per group
    a4 = orc.decode_reference_shared(q4, k, v, seq, b, K)
    for (bi, h), row in a4.items():
        assert row["idx"] == r[(bi, h // 4)]["idx"]


# ------------------------------------------------------------------------------------------
# Outer gate (R20)
# ------------------------------------------------------------------------------------------


def _outer_loss(qs, k, v, positions, b, selected, g, douts):
    return sum(float(np.dot(np.asarray(do), orc.outer_gated_row(q, k, v, int(i), b, selected,
                                                                   g)[0]))
               for q, i, do in zip(qs, positions, douts))


def test_outer_gate_unit_gates_give_plain_attention():
    rng = np.random.default_rng(95)
    n, d, b = 300, 16, 32
    q, k, v = rng.standard_normal(d), rng.standard_normal((n, d)), rng.standard_normal((n, d))
    sel = [1, 4, 6]
    o, lse = orc.outer_gated_row(q, k, v, 250, b, sel, {m: 1.0 for m in sel})
    ro, rl = orc.sparse_attention_row(q, k, v, 250, b, sel)
    assert np.allclose(o, ro, rtol=0, atol=1e-13) and abs(lse - rl) < 1e-13
    # scaling one block's gate by c adds (c - 1) times that block's weighted values, lse unchanged
    o2, lse2 = orc.outer_gated_row(q, k, v, 250, b, sel, {1: 1.0, 4: 3.0, 6: 1.0})
    assert abs(lse2 - rl) < 1e-13
    toks, owner = orc.token_set(250, b, sel, n)
    _, _, p = orc.attend(q, k, v, toks, np.zeros(len(toks)))
    part = sum(p[t] * v[toks[t]] for t, m in enumerate(owner) if m == 4)
    assert np.allclose(o2 - ro, 2.0 * part, rtol=0, atol=1e-12)


def test_outer_gate_gradient_matches_finite_differences():
    """The loss is linear in each outer gate, so a central difference recovers dg_m exactly
    (up to rounding); a planted sign error or a dropped block fails."""
    rng = np.random.default_rng(96)
    n, d, b = 256, 16, 32
    k, v = rng.standard_normal((n, d)), rng.standard_normal((n, d))
    positions = [192, 200, 223]
    qs = rng.standard_normal((3, d))
    douts = rng.standard_normal((3, d))
    sel = [0, 2, 5]
    g = {0: 0.2, 2: 0.5, 5: 0.3}
    dg = orc.gate_grad_rows_outer(qs, k, v, positions, b, sel, douts)
    for m in sel:
        h = 1e-3
        up = dict(g); up[m] += h
        dn = dict(g); dn[m] -= h
        fd = (_outer_loss(qs, k, v, positions, b, sel, up, douts)
              - _outer_loss(qs, k, v, positions, b, sel, dn, douts)) / (2 * h)
        assert abs(fd - dg[m]) < 1e-9 * max(1.0, abs(fd)), (m, fd, dg[m])


# ------------------------------------------------------------------------------------------
# FS-B forests and beam search (R21)
# ------------------------------------------------------------------------------------------


def test_fsb_forest_structure_and_node_summaries():
    """Trees per set bit of the cell count, largest first; a node's mean key is the mean of the
    raw keys below it (cells are full), its radius the largest leaf distance (brute force), its
    maximum norm and minimum position those of its leaves."""
    rng = np.random.default_rng(50)
    n, d, cell = 64 * 23, 8, 64
    k = rng.standard_normal((n, d))
    mean_k, max_norm, centre = orc.block_summaries(k, cell)
    for m in [1, 2, 3, 7, 8, 13, 23]:
        cells = list(range(m))
        nodes = orc.fsb_forest(cells, mean_k, max_norm, centre)
        roots = [(x["lo"], x["hi"]) for x in nodes if x["root"]]
        sizes = [1 << h for h in range(m.bit_length() - 1, -1, -1) if m & (1 << h)]
        assert [hi - lo for lo, hi in roots] == sizes
        assert roots[0][0] == 0 and all(a[1] == b[0] for a, b in zip(roots, roots[1:]))
        assert len(nodes) == sum(2 * s - 1 for s in sizes)
        for x in nodes:
            lo, hi = x["lo"], x["hi"]
            assert hi - lo == 1 << x["height"]
            toks = k[lo * cell:hi * cell]
            assert np.allclose(x["mu"], toks.mean(0), atol=1e-12)
            dist = np.linalg.norm(mean_k[lo:hi] - x["mu"], axis=1)
            assert abs(x["rho"] - (dist.max() if hi - lo > 1 else 0.0)) < 1e-12
            assert x["amax"] == max_norm[lo:hi].max() and x["pmin"] == centre[lo]
            if x["children"]:
                a, b = (nodes[j] for j in x["children"])
                assert (a["lo"], a["hi"], b["lo"], b["hi"]) == (lo, (lo + hi) // 2, (lo + hi) // 2, hi)


def test_fsb_node_bound_dominates_every_leaf_score():
    """U_v >= r_ic for every cell below v (equality at the leaves), for random queries, both
    forests, lambda > 0."""
    rng = np.random.default_rng(51)
    n, d, cell = 32 * 100, 16, 32
    k = rng.standard_normal((n, d)) * rng.uniform(0.5, 2.0, (n, 1))
    mean_k, max_norm, centre = orc.block_summaries(k, cell)
    for trial in range(6):
        q = rng.standard_normal(d) * 2
        i = int(rng.integers(100 * 32 - 200, 100 * 32))
        lam, sig = float(rng.uniform(0.1, 2.0)), float(rng.uniform(50, 3000))
        nc = orc.freesolo_num_candidates(i, cell, 128)
        r = orc.freesolo_scores(q, i, mean_k, max_norm, centre, lam, sig, nc)
        for cells in (list(range(nc)), orc.fsb_high_cells(max_norm, nc)):
            nodes = orc.fsb_forest(cells, mean_k, max_norm, centre)
            for x in nodes:
                below = cells[x["lo"]:x["hi"]]
                u = orc.fsb_bound(x, q, i, lam, sig)
                assert u >= max(r[c] for c in below) - 1e-12
                if x["height"] == 0:
                    assert abs(u - r[below[0]]) < 1e-12


def test_fsb_high_cells_are_those_at_or_above_the_median():
    rng = np.random.default_rng(52)
    for nc in [1, 2, 9, 10, 101, 400]:
        a = rng.standard_normal(500)
        got = orc.fsb_high_cells(a, nc)
        assert got == sorted(c for c in range(nc) if a[c] >= np.median(a[:nc]))
        assert len(got) == (nc + 1) // 2


def test_fsb_rerank_is_the_cells_log_sum_exp():
    rng = np.random.default_rng(53)
    n, d, cell = 32 * 20, 16, 32
    k, q = rng.standard_normal((n, d)), rng.standard_normal(d)
    cells = [0, 3, 19]
    got = orc.fsb_rerank_scores(q, k, cells, cell)
    for j, c in enumerate(cells):
        z = torch.as_tensor(k[c * cell:(c + 1) * cell]) @ torch.as_tensor(q) / math.sqrt(d)
        assert abs(got[j] - float(torch.logsumexp(z, 0))) < 1e-12


def test_fsb_beam_as_wide_as_the_forest_is_the_exhaustive_rerank():
    """A beam at least as wide as the cell count keeps every cell at every level, so the
    selection is the top K of the log-sum-exp re-rank over every candidate cell (full sort)."""
    rng = np.random.default_rng(54)
    n, d, cell = 32 * 64, 16, 32
    k = rng.standard_normal((n, d))
    summ = orc.block_summaries(k, cell)
    for i in [600, 1300, 2047]:
        q = rng.standard_normal(d)
        nc = orc.freesolo_num_candidates(i, cell, 128)
        sel, cand, _ = orc.fsb_select(q, i, k, summ, cell, 128, 4, 0.5, 300.0, width=nc)
        assert cand == list(range(nc))
        lse = [float(torch.logsumexp(torch.as_tensor(k[c * cell:(c + 1) * cell]) @
                                     torch.as_tensor(q) / math.sqrt(d), 0)) for c in range(nc)]
        want = sorted(sorted(range(nc), key=lambda c: (-lse[c], c))[:4])
        assert sel == want
    # a narrow beam reaches at most 2 x width cells and selects among them
    q = rng.standard_normal(d)
    sel, cand, _ = orc.fsb_select(q, 2047, k, summ, cell, 128, 4, 0.5, 300.0, width=2)
    assert len(cand) <= 4 and set(sel) <= set(cand)
