"""GPU parity: every call of the C ABI against the fp64 oracle on the same seeded inputs.

Tolerances (bf16 inputs with fp32 accumulation: 2e-2 on outputs, 1e-2 relative on dg; fp32
inputs: errors near 1e-6 over <= 2,000 terms, so 1e-4 still catches a wrong token or scale):
* block indices: bit-exact where the oracle's K-th and (K+1)-th scores differ by more than 1e-4
  relative; otherwise the GPU set must be one of the oracle's valid sets; bit-exact outright
  when the scores are supplied;
* outputs o: max abs error <= 2e-2 for bf16 inputs (fp32 accumulate), <= 1e-4 for fp32 inputs;
* lse: same bounds; dg: max |error| / max |dg| per query unit <= 1e-2 (bf16), 1e-4 (fp32).
"""
import math

import numpy as np
import pytest
import torch

import block_sparse_attention_summaries_b200 as bsa
from block_sparse_attention_summaries_b200 import inputs
from oracle import bsa_oracle as orc

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _lib(bsa_lib):
    return bsa_lib


def up(x, bf16):
    return torch.from_numpy(np.ascontiguousarray(x)).to(DEV, torch.bfloat16 if bf16 else
                                                         torch.float32)


def up_i32(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.int32)).to(DEV)


def tol(bf16):
    return 2e-2 if bf16 else 1e-4


def check_selection(gpu_idx, s, n_cand, K, exact):
    """Return the oracle's valid sets for this row and assert the GPU's is one of them."""
    gsel = sorted(int(x) for x in gpu_idx if x >= 0)
    if exact:
        ref = orc.topk_blocks(s, n_cand, K)
        assert gsel == ref, (gsel, ref)
        return [ref]
    sets = orc.valid_selections(s, n_cand, K)
    if sets is None:  # too many equivalent sets: check count and the clear part only
        assert len(gsel) == min(K, n_cand)
        return None
    assert gsel in sets, (gsel, sets[:3])
    return sets


# -------------------------------------------------------------------------------------------
# a1: summaries
# -------------------------------------------------------------------------------------------


@pytest.mark.parametrize("bf16", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_summaries(bf16, d):
    B, Hk, n, b = 2, 3, 1000, 64
    k = inputs.draw_normal(11, "k", (B, Hk, n, d), bf16) * 1.5 + 0.25
    if bf16:
        k = inputs.round_bf16(k)
    seq = np.array([1000, 777], dtype=np.int32)
    mean_k, mx, ce = bsa.build_block_summaries(up(k, bf16), b, up_i32(seq))
    torch.cuda.synchronize()
    mean_k, mx, ce = mean_k.cpu().numpy(), mx.cpu().numpy(), ce.cpu().numpy()
    C = (n + b - 1) // b
    for bi in range(B):
        L = seq[bi]
        for kh in range(Hk):
            rm, rx, rc = orc.block_summaries(k[bi, kh, :L], b)
            cl = len(rm)
            assert np.max(np.abs(mean_k[bi, kh, :cl] - rm)) < 1e-5
            assert np.max(np.abs(mx[bi, kh, :cl] - rx) / rx) < 1e-5
            assert np.array_equal(ce[bi, kh, :cl], rc.astype(np.float32))
            # blocks past the row's length: zero summary, centre of a full block
            for c in range(cl, C):
                assert not mean_k[bi, kh, c].any() and mx[bi, kh, c] == 0
                assert ce[bi, kh, c] == c * b + (b - 1) / 2


def test_summaries_append_current_block():
    B, Hk, n, d, b = 2, 2, 300, 128, 32
    k = inputs.draw_normal(12, "k", (B, Hk, n, d), True)
    seq = np.array([300, 129], dtype=np.int32)
    C = (n + b - 1) // b
    mean_k = torch.full((B, Hk, C, d), 7.0, device=DEV)
    mx = torch.full((B, Hk, C), 7.0, device=DEV)
    ce = torch.full((B, Hk, C), 7.0, device=DEV)
    bsa.build_block_summaries(up(k, True), b, up_i32(seq), -1, 1, mean_k, mx, ce)
    mean_k, mx = mean_k.cpu().numpy(), mx.cpu().numpy()
    for bi in range(B):
        cur = (seq[bi] - 1) // b
        for kh in range(Hk):
            rm, rx, _ = orc.block_summaries(k[bi, kh, :seq[bi]], b)
            assert np.max(np.abs(mean_k[bi, kh, cur] - rm[cur])) < 1e-5
            others = [c for c in range(C) if c != cur]
            assert (mean_k[bi, kh, others] == 7.0).all() and (mx[bi, kh, others] == 7.0).all()


# -------------------------------------------------------------------------------------------
# a2: decode scores
# -------------------------------------------------------------------------------------------


@pytest.mark.parametrize("G", [1, 4, 8])
@pytest.mark.parametrize("freesolo", [False, True])
def test_scores(G, freesolo):
    B, Hk, n, d, b = 2, 2, 2000, 128, 32
    Hq = Hk * G
    case = inputs.decode_case(13, B=B, Hq=Hq, Hk=Hk, d=d, n=n, b=b, K=4, needles=3,
                              seq_lens=[2000, 1111])
    k_gpu = up(case.k, True)
    mean_k, mx, ce = bsa.build_block_summaries(k_gpu, b, up_i32(case.seq_lens))
    lam = sig = None
    prefix = 0
    lam_np = np.linspace(0.2, 0.9, Hq).astype(np.float32)
    sig_np = np.linspace(100, 900, Hq).astype(np.float32)
    if freesolo:
        lam, sig, prefix = up(lam_np, False), up(sig_np, False), 128
    s, nc = bsa.score_blocks(up(case.q, True), mean_k, n, b, up_i32(case.seq_lens), mx, ce, lam,
                             sig, prefix)
    s, nc = s.cpu().numpy(), nc.cpu().numpy()
    for bi in range(B):
        L = case.seq_lens[bi]
        pos = L - 1
        for kh in range(Hk):
            rm, rx, rc = orc.block_summaries(case.k[bi, kh, :L], b)
            for g in range(G):
                h = kh * G + g
                if freesolo:
                    ncand = orc.freesolo_num_candidates(pos, b, 128)
                    ref = orc.freesolo_scores(case.q[bi, h], pos, rm, rx, rc, float(lam_np[h]),
                                              float(sig_np[h]), ncand)
                else:
                    ncand = orc.sas_num_candidates(pos, b)
                    ref = orc.dot_scores(case.q[bi, h], rm, ncand)
                assert nc[bi * Hq + h] == ncand
                assert np.max(np.abs(s[bi, h, :ncand] - ref)) < 2e-5 * max(1, np.abs(ref).max())
                assert np.isneginf(s[bi, h, ncand:]).all()


# -------------------------------------------------------------------------------------------
# a3: top-K (supplied scores: bit-exact)
# -------------------------------------------------------------------------------------------


@pytest.mark.parametrize("C,K", [(1, 1), (7, 3), (16, 4), (255, 15), (511, 15), (1000, 64),
                                 (4097, 31), (8191, 31), (16384, 256)])
def test_topk_exact(C, K):
    rows = 24
    rng = np.random.default_rng(C * 7 + K)
    s = rng.standard_normal((rows, C)).astype(np.float32)
    s[0] = np.round(s[0] * 2) / 2  # heavy ties
    s[1] = 0.0
    s[1, ::3] = -0.0  # signed zeros tie with +0
    if C > 4:
        s[2, rng.choice(C, size=C // 3, replace=False)] = np.nan
        s[3, : C // 2] = -np.inf
        s[4] = np.nan
    ncand = rng.integers(0, C + 1, size=rows).astype(np.int32)
    ncand[5] = C
    ncand[6] = 0
    ncand[7] = min(K, C)
    idx, cnt = bsa.topk_blocks(up(s, False), K, n_cand=up_i32(ncand))
    idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    for r in range(rows):
        ref = orc.topk_blocks(s[r].astype(np.float64), int(ncand[r]), K)
        assert cnt[r] == len(ref)
        assert list(idx[r, :len(ref)]) == ref, r
        assert (idx[r, len(ref):] == -1).all()


def test_topk_units_rule():
    B, Hq, U, C, qb, b, K = 1, 3, 40, 40, 64, 64, 5
    s = inputs.draw_normal(14, "s", (B, Hq, U, C), False)
    idx, cnt = bsa.topk_blocks(up(s, False), K, units=U, q_block=qb, b=b)
    idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    for h in range(Hq):
        for u in range(U):
            ref = orc.topk_blocks(s[0, h, u].astype(np.float64), (u * qb) // b, K)
            assert list(idx[0, h, u, :len(ref)]) == ref and cnt[0, h, u] == len(ref)


# -------------------------------------------------------------------------------------------
# a4: decode attention (tiny fp32 case with supplied scores, both modes)
# -------------------------------------------------------------------------------------------


@pytest.mark.parametrize("gate", [None, "selected", "all"])
def test_decode_tiny_supplied_scores(gate):
    case = inputs.tiny_decode_case(1000)
    B, Hq, d, n, b, K = case.B, case.Hq, case.d, case.n, case.b, case.K
    ref = orc.decode_reference(case.q, case.k, case.v, case.seq_lens, b, K, scores=case.scores,
                               gate_norm=gate)
    s_gpu = up(case.scores, False)
    ncand = up_i32(np.full(B * Hq, (n - 1) // b, np.int32))
    idx, cnt = bsa.topk_blocks(s_gpu, K, n_cand=ncand)
    o, lse = bsa.sparse_attn_fwd(up(case.q, False), up(case.k, False), up(case.v, False), idx, b,
                                 count=cnt, gate=gate is not None, norm=gate or "selected",
                                 scores=s_gpu)
    idx, o, lse = idx.cpu().numpy(), o.cpu().numpy(), lse.cpu().numpy()
    for h in range(Hq):
        r = ref[(0, h)]
        assert list(idx[0, h]) == r["idx"]
        assert np.max(np.abs(o[0, h] - r["o"])) < 1e-4
        assert abs(lse[0, h] - r["lse"]) < 1e-4


@pytest.mark.parametrize("G,K,b", [(4, 5, 64), (1, 3, 32), (8, 7, 128), (2, 40, 16)])
def test_decode_chain_ragged_bf16(G, K, b):
    B, Hk, n, d = 3, 2, 1500, 128
    Hq = Hk * G
    seq = [1500, 513, b]  # full, ragged, only the current block
    case = inputs.decode_case(15 + G, B=B, Hq=Hq, Hk=Hk, d=d, n=n, b=b, K=K, needles=4,
                              seq_lens=seq)
    k_gpu, v_gpu = up(case.k, True), up(case.v, True)
    sl = up_i32(case.seq_lens)
    mean_k, _, _ = bsa.build_block_summaries(k_gpu, b, sl)
    o, lse, idx = bsa.decode_step(up(case.q, True), k_gpu, v_gpu, mean_k, b, K, seq_lens=sl)
    o, lse, idx = o.float().cpu().numpy(), lse.cpu().numpy(), idx.cpu().numpy()
    summ = {}
    for bi in range(B):
        for h in range(Hq):
            kh = h // G
            L = int(seq[bi])
            if (bi, kh) not in summ:
                summ[(bi, kh)] = orc.block_summaries(case.k[bi, kh, :L], b)
            nc = orc.sas_num_candidates(L - 1, b)
            s = orc.round_f32(orc.dot_scores(case.q[bi, h], summ[(bi, kh)][0], nc))
            sets = check_selection(idx[bi, h], s, nc, K, exact=False)
            assert sets is not None
            outs = []
            for sel in sets:
                ro, rl = orc.sparse_attention_row(case.q[bi, h], case.k[bi, kh, :L],
                                                  case.v[bi, kh, :L], L - 1, b, sel)
                outs.append((np.max(np.abs(o[bi, h] - ro)), abs(lse[bi, h] - rl)))
            gsel = sorted(int(x) for x in idx[bi, h] if x >= 0)
            eo, el = outs[sets.index(gsel)]
            assert eo < 2e-2 and el < 2e-2, (bi, h, eo, el)


def test_decode_given_selection_cluster_path_matches_split_k():
    """bf16 K/V in 64-token blocks without a gate: bsa_sparse_attn_fwd (decode) runs the cluster
    step on the given selection.  Lists with repeats, negative and out-of-history entries and
    short counts: against the split-K kernel (the allocation-free entry) and the oracle over each
    row's distinct valid blocks."""
    B, Hq, Hk, n, d, b, K = 2, 8, 2, 4000, 128, 64, 9
    seq = [4000, 1234]
    case = inputs.decode_case(77, B=B, Hq=Hq, Hk=Hk, d=d, n=n, b=b, K=K, needles=2,
                              seq_lens=seq)
    q, k, v = up(case.q, True), up(case.k, True), up(case.v, True)
    sl = up_i32(case.seq_lens)
    rng = np.random.default_rng(5)
    idx = rng.integers(-2, 70, size=(B, Hq, K)).astype(np.int32)
    idx[0, 0, 1] = idx[0, 0, 0]
    idx[1, 3, :] = 5
    cnt = rng.integers(0, K + 1, size=(B, Hq)).astype(np.int32)
    cnt[0, 0] = K
    o1, lse1 = bsa.sparse_attn_fwd(q, k, v, up_i32(idx), b, count=up_i32(cnt), seq_lens=sl)
    o2, lse2 = bsa.sparse_attn_decode_noalloc(q, k, v, up_i32(idx), b, count=up_i32(cnt),
                                              seq_lens=sl)
    torch.cuda.synchronize()
    assert bsa.noalloc_status() == 0
    # the cluster step rounds the scaled query to bf16 for its MMAs: the bf16 output bar
    assert (o1.float() - o2.float()).abs().max().item() < 2e-2
    assert (lse1 - lse2).abs().max().item() < 1e-2
    o1, lse1 = o1.float().cpu().numpy(), lse1.cpu().numpy()
    G = Hq // Hk
    for bi in range(B):
        L = seq[bi]
        cur = (L - 1) // b
        for h in range(Hq):
            kh = h // G
            sel = sorted({int(m) for m in idx[bi, h, :cnt[bi, h]] if 0 <= m < cur})
            ro, rl = orc.sparse_attention_row(case.q[bi, h], case.k[bi, kh, :L],
                                              case.v[bi, kh, :L], L - 1, b, sel)
            assert np.max(np.abs(o1[bi, h] - ro)) < 2e-2, (bi, h)
            assert abs(lse1[bi, h] - rl) < 2e-2, (bi, h)


def test_decode_gated_bf16_all_history():
    B, Hq, Hk, n, d, b, K = 2, 8, 2, 2048, 128, 64, 6
    case = inputs.decode_case(16, B=B, Hq=Hq, Hk=Hk, d=d, n=n, b=b, K=K, needles=0,
                              supplied_scores=True, seq_lens=[2048, 1000])
    ref = {}
    for norm in ["selected", "all"]:
        ref = orc.decode_reference(case.q, case.k, case.v, case.seq_lens, b, K,
                                   scores=case.scores, gate_norm=norm)
        s_gpu = up(case.scores, False)
        ncand = up_i32(np.repeat((case.seq_lens - 1) // b, Hq))
        idx, cnt = bsa.topk_blocks(s_gpu, K, n_cand=ncand)
        o, lse = bsa.sparse_attn_fwd(up(case.q, True), up(case.k, True), up(case.v, True), idx, b,
                                     count=cnt, seq_lens=up_i32(case.seq_lens), gate=True,
                                     norm=norm, scores=s_gpu)
        o, lse, idx = o.float().cpu().numpy(), lse.cpu().numpy(), idx.cpu().numpy()
        for (bi, h), r in ref.items():
            assert list(idx[bi, h][:len(r["idx"])]) == r["idx"]
            assert np.max(np.abs(o[bi, h] - r["o"])) < 2e-2
            assert abs(lse[bi, h] - r["lse"]) < 2e-2


# -------------------------------------------------------------------------------------------
# a5 / a7: prefill attention and gate gradient
# -------------------------------------------------------------------------------------------


@pytest.mark.parametrize("gate", [None, "selected", "all"])
def test_prefill_tiny_per_query_selection(gate):
    """Tiny fp32 case: scores per query per block, so each query is its own unit."""
    case = inputs.tiny_decode_case(1000)  # q/k/v/s draws of the tiny case
    B, H, d, n, b, K = 1, 2, 64, 1024, 64, 4
    q = inputs.draw_normal(1000, "q_prefill", (B, H, n, d), False)
    s = inputs.draw_normal(1000, "s_prefill", (B, H, n, n // b), False)
    do = inputs.draw_normal(1000, "do_prefill", (B, H, n, d), False)
    k, v = case.k, case.v
    s_gpu = up(s, False)
    idx, cnt = bsa.topk_blocks(s_gpu, K, units=n, q_block=1, b=b)
    o, lse = bsa.sparse_attn_fwd(up(q, False), up(k, False), up(v, False), idx, b, count=cnt,
                                 q_block=1, gate=gate is not None, norm=gate or "selected",
                                 scores=s_gpu)
    dg = None
    if gate:
        dg = bsa.gate_grad(up(q, False), up(k, False), up(v, False), o, lse, up(do, False), idx, b,
                           s_gpu, q_block=1, count=cnt, norm=gate).cpu().numpy()
    o, lse, idx = o.cpu().numpy(), lse.cpu().numpy(), idx.cpu().numpy()
    rng = np.random.default_rng(3)
    rows = sorted(set([0, 1, 63, 64, 65, 127, 128, 255, 511, 1023]) |
                  set(rng.integers(0, n, 40).tolist()))
    for h in range(H):
        for i in rows:
            r = orc.prefill_unit_reference(q, k, v, s, b, 1, K, 0, h, i, gate, do)
            assert list(idx[0, h, i][:len(r["idx"])]) == r["idx"]
            assert np.max(np.abs(o[0, h, i] - r["o"][0])) < 1e-4
            assert abs(lse[0, h, i] - r["lse"][0]) < 1e-4
            if gate and len(r["idx"]):
                err = np.max(np.abs(dg[0, h, i, :len(r["idx"])] - r["dg"]))
                assert err <= 1e-4 * max(1e-3, np.max(np.abs(r["dg"]))), (h, i, err)


@pytest.mark.parametrize("gate", [None, "selected", "all"])
def test_prefill_bf16_units(gate):
    B, Hq, Hk, n, d, b, K = 1, 4, 2, 1024 + 37, 128, 64, 6
    case = inputs.prefill_case(17, B=B, Hq=Hq, Hk=Hk, d=d, n=n, b=b, K=K, q_block=64)
    s_gpu = up(case.scores, False)
    q, k, v = up(case.q, True), up(case.k, True), up(case.v, True)
    idx, cnt = bsa.topk_blocks(s_gpu, K, units=case.U, q_block=64, b=b)
    o, lse = bsa.sparse_attn_fwd(q, k, v, idx, b, count=cnt, q_block=64, gate=gate is not None,
                                 norm=gate or "selected", scores=s_gpu)
    dg = None
    if gate:
        dg = bsa.gate_grad(q, k, v, o, lse, up(case.dout, True), idx, b, s_gpu, q_block=64,
                           count=cnt, norm=gate).cpu().numpy()
    o, lse, idx = o.float().cpu().numpy(), lse.cpu().numpy(), idx.cpu().numpy()
    for h in range(Hq):
        for u in [0, 1, 2, 5, 9, 15, 16]:
            r = orc.prefill_unit_reference(case.q, case.k, case.v, case.scores, b, 64, K, 0, h, u,
                                           gate, case.dout)
            lo = u * 64
            assert list(idx[0, h, u][:len(r["idx"])]) == r["idx"]
            assert np.max(np.abs(o[0, h, lo:lo + len(r["o"])] - r["o"])) < 2e-2
            assert np.max(np.abs(lse[0, h, lo:lo + len(r["o"])] - r["lse"])) < 2e-2
            if gate and len(r["idx"]):
                err = np.max(np.abs(dg[0, h, u, :len(r["idx"])] - r["dg"]))
                assert err <= 1e-2 * np.max(np.abs(r["dg"])), (h, u, err)


# -------------------------------------------------------------------------------------------
# selector gradient through the log-softmax gate
# -------------------------------------------------------------------------------------------


@pytest.mark.parametrize("norm", ["selected", "all"])
def test_selector_grad_rows(norm):
    """ds from given dg: fp32 kernel against the fp64 chain rule, rows with no, few and many
    candidates, K up to 32."""
    rng = np.random.default_rng(31)
    rows, C = 300, 200
    s = rng.standard_normal((rows, C)).astype(np.float32) * 2.0
    n_cand = rng.integers(0, C + 1, rows).astype(np.int32)
    n_cand[:4] = [0, 1, 3, C]
    for K in (5, 32):
        idx = np.full((rows, K), -1, np.int32)
        dg = np.zeros((rows, K), np.float32)
        for r in range(rows):
            sel = orc.topk_blocks(s[r].astype(np.float64), int(n_cand[r]), K)
            idx[r, :len(sel)] = sel
            dg[r, :len(sel)] = rng.standard_normal(len(sel))
        ds = bsa.selector_grad(up(s, False), up_i32(n_cand), up_i32(idx), None,
                               up(dg, False), bsa.NORM_SELECTED if norm == "selected"
                               else bsa.NORM_ALL_HISTORY).cpu().numpy()
        for r in range(rows):
            nc = int(n_cand[r])
            sel = [int(m) for m in idx[r] if m >= 0]
            ref = orc.selector_grad_row(s[r].astype(np.float64), nc, sel,
                                        {m: float(dg[r, j]) for j, m in enumerate(sel)}, norm)
            scale = max(1.0, float(np.max(np.abs(ref))) if nc else 1.0)
            assert np.max(np.abs(ds[r, :nc] - ref), initial=0.0) <= 1e-5 * scale, (K, r)
            assert np.all(ds[r, nc:] == 0.0)


@pytest.mark.parametrize("norm", ["selected", "all"])
def test_selector_grad_chain_bf16_units(norm):
    """The training backward o -> g -> s on bf16 units: GPU dg then GPU ds against the oracle's
    gate gradient and chain rule on sampled units."""
    B, Hq, Hk, n, d, b, K = 1, 4, 2, 1024 + 37, 128, 64, 6
    case = inputs.prefill_case(17, B=B, Hq=Hq, Hk=Hk, d=d, n=n, b=b, K=K, q_block=64)
    s_gpu = up(case.scores, False)
    q, k, v = up(case.q, True), up(case.k, True), up(case.v, True)
    idx, cnt = bsa.topk_blocks(s_gpu, K, units=case.U, q_block=64, b=b)
    o, lse = bsa.sparse_attn_fwd(q, k, v, idx, b, count=cnt, q_block=64, gate=True, norm=norm,
                                 scores=s_gpu)
    dg = bsa.gate_grad(q, k, v, o, lse, up(case.dout, True), idx, b, s_gpu, q_block=64,
                       count=cnt, norm=norm)
    n_cand = torch.arange(case.U, dtype=torch.int32, device=DEV).expand(B, Hq, case.U)
    ds = bsa.selector_grad(s_gpu, n_cand.contiguous(), idx, cnt, dg,
                           bsa.NORM_SELECTED if norm == "selected" else bsa.NORM_ALL_HISTORY)
    ds = ds.cpu().numpy()
    for h in range(Hq):
        for u in [1, 2, 5, 9, 15, 16]:
            r = orc.prefill_unit_reference(case.q, case.k, case.v, case.scores, b, 64, K, 0, h, u,
                                           norm, case.dout)
            sel = r["idx"]
            dgr = {m: float(x) for m, x in zip(sel, r["dg"])}
            ref = orc.selector_grad_row(case.scores[0, h, u].astype(np.float64), u, sel, dgr, norm)
            err = np.max(np.abs(ds[0, h, u, :u] - ref))
            assert err <= 1e-2 * max(1e-6, np.max(np.abs(ref))), (h, u, err)


# -------------------------------------------------------------------------------------------
# failure path
# -------------------------------------------------------------------------------------------


def test_bounded_wait_reports_timeout_and_context_survives():
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    assert bsa.workspace_status(ws) == 0
    bsa.selftest_bounded_wait(ws, polls=200)
    assert bsa.workspace_status(ws) == 6  # BSA_ERR_TIMEOUT, then cleared
    assert bsa.workspace_status(ws) == 0
    x = torch.ones(4, device=DEV) * 2  # the context still runs work
    assert float(x.sum()) == 8.0


def test_errors_on_device_tensors():
    k = torch.zeros(1, 1, 64, 96, device=DEV, dtype=torch.bfloat16)
    with pytest.raises(bsa.BsaError) as e:
        bsa.build_block_summaries(k, 16)
    assert e.value.code == 4


@pytest.mark.parametrize("d", [64, 128])
def test_prefill_bf16_tensor_core_shapes(d):
    """bf16, 64-query units over 64-token blocks, even GQA groups: the tcgen05 kernel's shapes."""
    B, Hq, Hk, n, b, K = 2, 8, 2, 2048 + 21, 64, 9
    case = inputs.prefill_case(18 + d, B=B, Hq=Hq, Hk=Hk, d=d, n=n, b=b, K=K, q_block=64)
    s_gpu = up(case.scores, False)
    q, k, v = up(case.q, True), up(case.k, True), up(case.v, True)
    idx, cnt = bsa.topk_blocks(s_gpu, K, units=case.U, q_block=64, b=b)
    for gate in [None, "selected", "all"]:
        o, lse = bsa.sparse_attn_fwd(q, k, v, idx, b, count=cnt, q_block=64,
                                     gate=gate is not None, norm=gate or "selected", scores=s_gpu)
        o, lse = o.float().cpu().numpy(), lse.cpu().numpy()
        for bi in range(B):
            for h in [0, 3, 4, 7]:
                for u in [0, 1, 8, 9, 17, 31, case.U - 1]:
                    r = orc.prefill_unit_reference(case.q, case.k, case.v, case.scores, b, 64, K,
                                                   bi, h, u, gate)
                    lo = u * 64
                    m = len(r["o"])
                    assert np.max(np.abs(o[bi, h, lo:lo + m] - r["o"])) < 2e-2, (gate, bi, h, u)
                    assert np.max(np.abs(lse[bi, h, lo:lo + m] - r["lse"])) < 2e-2


def test_prefill_gated_full_size_sampled():
    """The SAS training-mode prefill workload (batch 2, 32/8 heads, d = 128, 16K context, top-16
    blocks per 64-query unit, log-softmax gate over the selected blocks): output, lse and the
    gate gradient on sampled units."""
    case = inputs.prefill_case(5000)
    s_gpu = up(case.scores, False)
    q, k, v = up(case.q, True), up(case.k, True), up(case.v, True)
    idx, cnt = bsa.topk_blocks(s_gpu, case.K, units=case.U, q_block=64, b=64)
    o, lse = bsa.sparse_attn_fwd(q, k, v, idx, 64, count=cnt, q_block=64, gate=True,
                                 norm="selected", scores=s_gpu)
    dg = bsa.gate_grad(q, k, v, o, lse, up(case.dout, True), idx, 64, s_gpu, q_block=64,
                       count=cnt, norm="selected")
    o, lse, dg, idx = (x.float().cpu().numpy() if x.dtype != torch.int32 else x.cpu().numpy()
                       for x in (o, lse, dg, idx))
    rng = np.random.default_rng(11)
    units = [(0, 0, 0), (1, 31, 255), (0, 5, 16), (1, 12, 17)] + \
        [(int(a), int(c), int(e)) for a, c, e in zip(rng.integers(0, 2, 8),
                                                     rng.integers(0, 32, 8),
                                                     rng.integers(0, 256, 8))]
    for bi, h, u in units:
        r = orc.prefill_unit_reference(case.q, case.k, case.v, case.scores, 64, 64, case.K, bi, h,
                                       u, "selected", case.dout)
        lo = u * 64
        assert list(idx[bi, h, u][:len(r["idx"])]) == r["idx"]
        assert np.max(np.abs(o[bi, h, lo:lo + 64] - r["o"])) < 2e-2, (bi, h, u)
        assert np.max(np.abs(lse[bi, h, lo:lo + 64] - r["lse"])) < 2e-2
        if len(r["idx"]):
            err = np.max(np.abs(dg[bi, h, u, :len(r["idx"])] - r["dg"]))
            assert err <= 1e-2 * np.max(np.abs(r["dg"])), (bi, h, u, err)


# -------------------------------------------------------------------------------------------
# outer gate (the gate outside the softmax): forward and gradient, fp32 on the row kernels and
# bf16 units on the tensor cores
# -------------------------------------------------------------------------------------------


@pytest.mark.parametrize("norm", ["selected", "all"])
def test_prefill_outer_gate_fp32_per_query(norm):
    case = inputs.tiny_decode_case(1000)
    B, H, d, n, b, K = 1, 2, 64, 1024, 64, 4
    q = inputs.draw_normal(1000, "q_prefill", (B, H, n, d), False)
    s = inputs.draw_normal(1000, "s_prefill", (B, H, n, n // b), False)
    do = inputs.draw_normal(1000, "do_prefill", (B, H, n, d), False)
    k, v = case.k, case.v
    s_gpu = up(s, False)
    qg, kg, vg = up(q, False), up(k, False), up(v, False)
    idx, cnt = bsa.topk_blocks(s_gpu, K, units=n, q_block=1, b=b)
    o, lse = bsa.sparse_attn_fwd(qg, kg, vg, idx, b, count=cnt, q_block=1, gate="outer",
                                 norm=norm, scores=s_gpu)
    dg = bsa.gate_grad(qg, kg, vg, o, lse, up(do, False), idx, b, s_gpu, q_block=1, count=cnt,
                       norm=norm, outer=True).cpu().numpy()
    o, lse = o.cpu().numpy(), lse.cpu().numpy()
    rng = np.random.default_rng(4)
    rows = sorted(set([0, 63, 64, 65, 255, 1023]) | set(rng.integers(0, n, 30).tolist()))
    for h in range(H):
        for i in rows:
            r = orc.prefill_unit_reference_outer(q, k, v, s, b, 1, K, 0, h, i, norm, do)
            assert np.max(np.abs(o[0, h, i] - r["o"][0])) < 1e-4, (h, i)
            assert abs(lse[0, h, i] - r["lse"][0]) < 1e-4, (h, i)
            if len(r["idx"]):
                err = np.max(np.abs(dg[0, h, i, :len(r["idx"])] - r["dg"]))
                assert err <= 1e-4 * max(1e-3, np.max(np.abs(r["dg"]))), (h, i, err)


def test_prefill_outer_gate_bf16_units():
    """bf16 units of 64 queries on the tensor-core forward and gradient: forward and dg against
    the oracle on sampled units."""
    B, Hq, Hk, n, d, b, K = 1, 4, 2, 1024 + 37, 128, 64, 6
    case = inputs.prefill_case(17, B=B, Hq=Hq, Hk=Hk, d=d, n=n, b=b, K=K, q_block=64)
    s_gpu = up(case.scores, False)
    q, k, v = up(case.q, True), up(case.k, True), up(case.v, True)
    idx, cnt = bsa.topk_blocks(s_gpu, K, units=case.U, q_block=64, b=b)
    o, lse = bsa.sparse_attn_fwd(q, k, v, idx, b, count=cnt, q_block=64, gate="outer",
                                 norm="all", scores=s_gpu)
    dg = bsa.gate_grad(q, k, v, o, lse, up(case.dout, True), idx, b, s_gpu, q_block=64,
                       count=cnt, norm="all", outer=True).cpu().numpy()
    o, lse = o.float().cpu().numpy(), lse.cpu().numpy()
    for h in range(Hq):
        for u in [0, 1, 5, 9, 16]:
            r = orc.prefill_unit_reference_outer(case.q, case.k, case.v, case.scores, b, 64, K, 0,
                                                 h, u, "all", case.dout)
            lo = u * 64
            assert np.max(np.abs(o[0, h, lo:lo + len(r["o"])] - r["o"])) < 2e-2, (h, u)
            assert np.max(np.abs(lse[0, h, lo:lo + len(r["o"])] - r["lse"])) < 2e-2, (h, u)
            if len(r["idx"]):
                err = np.max(np.abs(dg[0, h, u, :len(r["idx"])] - r["dg"]))
                assert err <= 1e-2 * np.max(np.abs(r["dg"])), (h, u, err)


def test_outer_gate_decode_unsupported():
    case = inputs.tiny_decode_case(1000)
    q = up(case.q, False)
    idx = torch.zeros(q.shape[0], q.shape[1], 2, dtype=torch.int32, device=DEV)
    with pytest.raises(bsa.BsaError) as e:
        bsa.sparse_attn_fwd(q, up(case.k, False), up(case.v, False), idx, 64, gate="outer",
                            scores=torch.zeros(q.shape[0], q.shape[1], 64, device=DEV))
    assert e.value.code == 4
