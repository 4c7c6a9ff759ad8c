"""GPU parity of the fused single-launch decode step (bsa_decode_step).

Checked three ways: against the fp64 oracle (selection by the near-tie rule, outputs within the
bf16 bar of 2e-2), against the chain of separate calls on the GPU (which computes the scores with
the same arithmetic, so the selected indices must be identical), and for the summary append.
"""
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


def upload(case):
    dt = torch.bfloat16 if case.bf16 else torch.float32
    q, k, v = (torch.from_numpy(x).to(DEV, dt) for x in (case.q, case.k, case.v))
    sl = torch.from_numpy(case.seq_lens).to(DEV)
    return q, k, v, sl


def oracle_check(case, idx, o, lse, rows, tol):
    summ = {}
    G = case.Hq // case.Hk
    for bi, h in rows:
        kh = h // G
        L = int(case.seq_lens[bi])
        if (bi, kh) not in summ:
            summ[(bi, kh)] = orc.block_summaries(case.k[bi, kh, :L], case.b)
        nc = orc.sas_num_candidates(L - 1, case.b)
        s = orc.round_f32(orc.dot_scores(case.q[bi, h], summ[(bi, kh)][0], nc))
        sets = orc.valid_selections(s, nc, case.K)
        gsel = sorted(int(x) for x in idx[bi, h] if x >= 0)
        assert sets is not None and gsel in sets, (bi, h, gsel)
        ro, rl = orc.sparse_attention_row(case.q[bi, h], case.k[bi, kh, :L], case.v[bi, kh, :L],
                                          L - 1, case.b, gsel)
        assert np.max(np.abs(o[bi, h] - ro)) < tol, (bi, h)
        assert abs(lse[bi, h] - rl) < tol, (bi, h)


@pytest.mark.parametrize("G,K,b,d,bf16", [(4, 15, 64, 128, True), (1, 3, 32, 64, True),
                                          (8, 7, 128, 128, True), (2, 31, 16, 64, True),
                                          (4, 5, 64, 128, False), (8, 32, 64, 64, True)])
def test_fused_matches_chain_and_oracle(G, K, b, d, bf16):
    Hk, n = 2, 3000
    seq = [3000, 1025, b, 777]
    case = inputs.decode_case(50 + G + K, B=4, Hq=Hk * G, Hk=Hk, d=d, n=n, b=b, K=K, needles=5,
                              bf16=bf16, seq_lens=seq)
    q, k, v, sl = upload(case)
    mean_k, _, _ = bsa.build_block_summaries(k, b, sl)
    o1, lse1, idx1, cnt1 = bsa.decode_step_fused(q, k, v, mean_k, b, K, seq_lens=sl, append=False)
    o2, lse2, idx2 = bsa.decode_step(q, k, v, mean_k, b, K, seq_lens=sl, append=False)
    torch.cuda.synchronize()
    assert torch.equal(idx1, idx2), "fused and separate selections differ"
    assert (o1.float() - o2.float()).abs().max().item() < (1e-2 if bf16 else 1e-5)
    rows = [(bi, h) for bi in range(4) for h in range(case.Hq)]
    oracle_check(case, idx1.cpu().numpy(), o1.float().cpu().numpy(), lse1.cpu().numpy(), rows,
                 2e-2 if bf16 else 1e-4)
    exp_cnt = np.minimum(K, (case.seq_lens - 1) // b)
    assert (cnt1.cpu().numpy() == exp_cnt[:, None]).all()


def test_fused_appends_current_block_summary():
    case = inputs.decode_case(61, B=3, Hq=8, Hk=2, d=128, n=2000, b=64, K=6, needles=3,
                              seq_lens=[2000, 1100, 64])
    q, k, v, sl = upload(case)
    mean_k, mx, ce = bsa.build_block_summaries(k, 64, sl)
    ref_m, ref_x, ref_c = mean_k.clone(), mx.clone(), ce.clone()
    cur = (sl - 1) // 64
    for bi in range(3):  # spoil the current block's summary; the step must restore it
        mean_k[bi, :, cur[bi]] = 99.0
        mx[bi, :, cur[bi]] = 99.0
        ce[bi, :, cur[bi]] = 99.0
    bsa.decode_step_fused(q, k, v, mean_k, 64, 6, seq_lens=sl, append=True, max_norm=mx, centre=ce)
    torch.cuda.synchronize()
    assert (mean_k - ref_m).abs().max().item() < 1e-5
    assert ((mx - ref_x).abs() / ref_x.clamp_min(1e-6)).max().item() < 1e-5
    assert torch.equal(ce, ref_c)


def test_fused_freesolo_bias_matches_separate_scoring():
    case = inputs.decode_case(62, B=2, Hq=8, Hk=2, d=64, n=4096, b=32, K=4, needles=4)
    q, k, v, sl = upload(case)
    lam = torch.linspace(0.2, 0.9, 8, device=DEV)
    sig = torch.linspace(100, 900, 8, device=DEV)
    mean_k, mx, ce = bsa.build_block_summaries(k, 32, sl)
    _, _, idx1, cnt1 = bsa.decode_step_fused(q, k, v, mean_k, 32, 4, seq_lens=sl, append=False,
                                             max_norm=mx, centre=ce, lambda_h=lam, sigma_h=sig,
                                             prefix_block=128)
    s, nc = bsa.score_blocks(q, mean_k, case.n, 32, sl, mx, ce, lam, sig, 128)
    idx2, cnt2 = bsa.topk_blocks(s, 4, n_cand=nc)
    torch.cuda.synchronize()
    assert torch.equal(idx1, idx2) and torch.equal(cnt1, cnt2.view_as(cnt1))


@pytest.mark.parametrize("wl", ["sas_gqa_decode_32k", "long_decode_512k"])
def test_fused_full_size(wl):
    """Full decode workloads (32K context x batch 8; 512K context): every row against the separate
    calls, sampled rows against the oracle."""
    w = dict(sas_gqa_decode_32k=dict(seed=2000, B=8, n=32768, K=15, needles=16,
                                     needle_layout="random"),
             long_decode_512k=dict(seed=3000, B=1, n=524288, K=31, needles=64,
                                   needle_layout="stride"))[wl]
    case = inputs.decode_case(w["seed"], B=w["B"], Hq=32, Hk=8, d=128, n=w["n"], b=64, K=w["K"],
                              needles=w["needles"], needle_layout=w["needle_layout"])
    q, k, v, sl = upload(case)
    mean_k, _, _ = bsa.build_block_summaries(k, 64)
    o1, lse1, idx1, cnt1 = bsa.decode_step_fused(q, k, v, mean_k, 64, w["K"], append=False)
    o2, lse2, idx2 = bsa.decode_step(q, k, v, mean_k, 64, w["K"], append=False)
    # with a workspace: two launches at 512K (chunk Top-K over the whole GPU, then the merge),
    # one launch at 32K; the same selection either way
    need = bsa.decode_step_workspace_bytes(w["B"], 32, 8, w["n"], 128, 64, w["K"])
    assert (need > 0) == (w["n"] // 64 > 512)
    o3, lse3, idx3, cnt3 = bsa.decode_step_ws(q, k, v, mean_k, 64, w["K"], append=False)
    torch.cuda.synchronize()
    assert torch.equal(idx1, idx2)
    assert torch.equal(idx3, idx1) and torch.equal(cnt3, cnt1)
    assert (o1.float() - o2.float()).abs().max().item() < 1e-2
    assert (o3.float() - o1.float()).abs().max().item() < 1e-2
    assert (lse3 - lse1).abs().max().item() < 1e-3
    if w["B"] == 1:  # long context: every head of the sequence
        rows = [(0, h) for h in range(32)]
    else:
        rng = np.random.default_rng(7)
        rows = sorted({(int(bi), int(h)) for bi, h in zip(rng.integers(0, w["B"], 16),
                                                            rng.integers(0, 32, 16))} | {(0, 0)})
    oracle_check(case, idx1.cpu().numpy(), o1.float().cpu().numpy(), lse1.cpu().numpy(), rows,
                 2e-2)
    # needle recall: every head of a group sees its planted blocks first
    idx_np = idx1.cpu().numpy()
    hits = tot = 0
    for (bi, kh), blocks in case.needles.items():
        sel = set(idx_np[bi, kh * 4:(kh + 1) * 4].ravel().tolist())
        hits += len(sel & set(int(c) for c in blocks))
        tot += len(blocks)
    assert hits / tot > 0.9


@pytest.mark.parametrize("n,B", [(40000, 2), (64 * 513 + 10, 1)])
def test_fused_long_history_local_and_merged_selection(n, B):
    """More than 512 history blocks: each CTA selects its slice's Top-K and the cluster merges the
    candidates (some CTAs of the cluster hold no block at all); every row against the separate
    calls and sampled rows against the oracle."""
    case = inputs.decode_case(64 + B, B=B, Hq=8, Hk=2, d=128, n=n, b=64, K=13, needles=9,
                              seq_lens=[n, n - 3000][:B])
    q, k, v, sl = upload(case)
    mean_k, _, _ = bsa.build_block_summaries(k, 64, sl)
    o1, lse1, idx1, cnt1 = bsa.decode_step_fused(q, k, v, mean_k, 64, 13, seq_lens=sl,
                                                 append=False)
    o2, lse2, idx2 = bsa.decode_step(q, k, v, mean_k, 64, 13, seq_lens=sl, append=False)
    o3, lse3, idx3, cnt3 = bsa.decode_step_ws(q, k, v, mean_k, 64, 13, seq_lens=sl,
                                              append=False)  # chunk Top-K + merge launches
    torch.cuda.synchronize()
    assert torch.equal(idx1, idx2)
    assert torch.equal(idx3, idx1) and torch.equal(cnt3, cnt1)
    assert (o1.float() - o2.float()).abs().max().item() < 1e-2
    assert (o3.float() - o1.float()).abs().max().item() < 1e-2
    rows = [(bi, h) for bi in range(B) for h in (0, 3, 5, 7)]
    oracle_check(case, idx1.cpu().numpy(), o1.float().cpu().numpy(), lse1.cpu().numpy(), rows,
                 2e-2)


@pytest.mark.parametrize("C", [300, 1000])
def test_fused_all_scores_tied_take_the_lowest_blocks(C):
    """Every history block scores exactly 0 (all keys zero): the Top-K is the K lowest block
    indices for every head, on the whole-row path (300 blocks) and on the local + merge path
    (1000 blocks); the threshold pass leaves every key as a candidate, so the radix select runs."""
    B, Hk, G, d, b, K = 2, 2, 4, 64, 64, 11
    n = C * b
    k = torch.zeros(B, Hk, n, d, device=DEV, dtype=torch.bfloat16)
    g = torch.Generator(device=DEV).manual_seed(5)
    v = torch.randn(B, Hk, n, d, device=DEV, generator=g).to(torch.bfloat16)
    q = torch.randn(B, Hk * G, d, device=DEV, generator=g).to(torch.bfloat16)
    mean_k, _, _ = bsa.build_block_summaries(k, b)
    o1, _, idx1, cnt1 = bsa.decode_step_fused(q, k, v, mean_k, b, K, append=False)
    o2, _, idx2 = bsa.decode_step(q, k, v, mean_k, b, K, append=False)
    torch.cuda.synchronize()
    want = torch.arange(K, device=DEV, dtype=torch.int32).expand(B, Hk * G, K)
    assert torch.equal(idx1, want) and torch.equal(idx2, want)
    assert torch.equal(cnt1, torch.full_like(cnt1, K))
    # zero keys: every attended token has logit 0, so o is the mean of the attended values
    vf = v.float()
    cur = (n - 1) // b
    for bi in range(B):
        for kh in range(Hk):
            toks = torch.cat([vf[bi, kh, :K * b], vf[bi, kh, cur * b:n]])
            ref = toks.mean(0)
            for h in range(kh * G, (kh + 1) * G):
                assert (o1[bi, h].float() - ref).abs().max().item() < 2e-2
    assert (o1.float() - o2.float()).abs().max().item() < 1e-2


@pytest.mark.parametrize("C,K", [(1000, 11), (4096, 32)])
def test_workspace_path_all_scores_tied_take_the_lowest_blocks(C, K):
    """The two-launch path with every score tied: each chunk keeps its K lowest blocks, every
    chunk threshold equals the common key, so every kept entry survives the bound; at 4096 blocks
    (32 chunks x 32 entries) the survivors overflow one merge buffer and the running Top-K keeps
    the lowest blocks.  The result is the K lowest block indices, as on the one-launch path."""
    B, Hk, G, d, b = 1, 2, 4, 64, 64
    n = C * b + 17
    k = torch.zeros(B, Hk, n, d, device=DEV, dtype=torch.bfloat16)
    g = torch.Generator(device=DEV).manual_seed(6)
    v = torch.randn(B, Hk, n, d, device=DEV, generator=g).to(torch.bfloat16)
    q = torch.randn(B, Hk * G, d, device=DEV, generator=g).to(torch.bfloat16)
    mean_k, _, _ = bsa.build_block_summaries(k, b)
    assert bsa.decode_step_workspace_bytes(B, Hk * G, Hk, n, d, b, K) > 0
    o1, lse1, idx1, cnt1 = bsa.decode_step_ws(q, k, v, mean_k, b, K, append=False)
    o2, lse2, idx2, cnt2 = bsa.decode_step_fused(q, k, v, mean_k, b, K, append=False)
    torch.cuda.synchronize()
    want = torch.arange(K, device=DEV, dtype=torch.int32).expand(B, Hk * G, K)
    assert torch.equal(idx1, want) and torch.equal(idx2, want)
    assert torch.equal(cnt1, torch.full_like(cnt1, K))
    assert (o1.float() - o2.float()).abs().max().item() < 1e-2


@pytest.mark.parametrize("n,B,K,extra", [(2048 + 17, 2, 7, 0), (600 * 64 + 5, 1, 13, 0),
                                         (2048 + 17, 2, 7, 1), (600 * 64 + 5, 1, 13, 2)])
def test_host_io_step_matches_device_buffers(n, B, K, extra):
    """DECODE_HOST_IO: q and o in page-locked host memory, the step staging q itself and writing o
    to host memory (one launch at 32 history blocks, two past 512; alone, with the shared
    selection and with bf16 summaries), against the same step on device buffers; two calls in a
    row check that the staging is reused safely."""
    Hq, Hk, d, b = 8, 2, 128, 64
    case = inputs.decode_case(90 + B, B=B, Hq=Hq, Hk=Hk, d=d, n=n, b=b, K=K, needles=3)
    q, k, v, sl = upload(case)
    mean_k, _, _ = bsa.build_block_summaries(k, b)
    xf = {0: 0, 1: bsa.DECODE_SHARED_SELECTION, 2: bsa.DECODE_BF16_SUMMARIES}[extra]
    if xf & bsa.DECODE_BF16_SUMMARIES:
        mean_k = bsa.round_summaries_bf16(mean_k)
    flags = bsa.DECODE_HOST_IO | xf
    ws = torch.empty(bsa.decode_step_workspace_bytes(B, Hq, Hk, n, d, b, K, flags),
                     dtype=torch.uint8, device=DEV)
    q2 = (q * 0.5).contiguous()
    outs = []
    for qq in (q, q2):
        q_host = qq.cpu().pin_memory()
        o_host = torch.full((B, Hq, d), float("nan"), dtype=torch.bfloat16).pin_memory()
        o1, lse1, idx1, cnt1 = bsa.decode_step_ws(q_host, k, v, mean_k, b, K, flags=flags, ws=ws,
                                                  o=o_host, append=False)
        outs.append((o1, lse1.clone(), idx1.clone()))
    torch.cuda.synchronize()
    for qq, (o1, lse1, idx1) in zip((q, q2), outs):
        o2, lse2, idx2, _ = bsa.decode_step_ws(qq, k, v, mean_k, b, K, flags=xf, append=False)
        torch.cuda.synchronize()
        assert not o1.is_cuda and torch.isfinite(o1.float()).all()
        assert torch.equal(idx1, idx2)
        assert (o1.float() - o2.float().cpu()).abs().max().item() < 1e-2
        assert (lse1 - lse2).abs().max().item() < 1e-3


def test_workspace_too_small_is_refused():
    n, b, K = 600 * 64, 64, 8
    need = bsa.decode_step_workspace_bytes(1, 8, 2, n, 128, b, K)
    assert need > 0
    q = torch.randn(1, 8, 128, device=DEV).to(torch.bfloat16)
    k = torch.randn(1, 2, n, 128, device=DEV).to(torch.bfloat16)
    mean_k, _, _ = bsa.build_block_summaries(k, b)
    ws = torch.empty(need - 16, dtype=torch.uint8, device=DEV)
    with pytest.raises(bsa.BsaError):
        bsa.decode_step_ws(q, k, k, mean_k, b, K, ws=ws, append=False)


# ---- variants: GQA-shared selection and bf16 summaries (bsa_decode_step_ex) ------------------


def test_round_summaries_bf16_bit_exact():
    rng = np.random.default_rng(70)
    x = (rng.standard_normal(100_003) * 10.0 ** rng.integers(-20, 20, 100_003)).astype(np.float32)
    grid = orc.round_bf16(x[:4000]).astype(np.float32)     # ties: halfway between grid points
    x[:4000] = grid + np.float32(2.0 ** -8) * np.abs(grid)
    x[-5:] = [np.inf, -np.inf, np.nan, 0.0, np.finfo(np.float32).max]
    out = bsa.round_summaries_bf16(torch.from_numpy(x).to(DEV))
    torch.cuda.synchronize()
    got = out.float().cpu().numpy().astype(np.float64)
    ref = orc.round_bf16(x)
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all(), np.flatnonzero(~same)[:5]


def shared_oracle_check(case, idx, o, lse, summaries=None):
    ref = orc.decode_reference_shared(case.q, case.k, case.v, case.seq_lens, case.b, case.K,
                                      summaries=summaries)
    G = case.Hq // case.Hk
    for (bi, h), r in ref.items():
        L = int(case.seq_lens[bi])
        nc = orc.sas_num_candidates(L - 1, case.b)
        sets = orc.valid_selections(r["scores"], nc, case.K)
        gsel = sorted(int(x) for x in idx[bi, h] if x >= 0)
        assert sets is not None and gsel in sets, (bi, h, gsel)
        # every head of the group holds the group's selection
        assert gsel == sorted(int(x) for x in idx[bi, (h // G) * G] if x >= 0)
        kh = h // G
        ro, rl = orc.sparse_attention_row(case.q[bi, h], case.k[bi, kh, :L], case.v[bi, kh, :L],
                                          L - 1, case.b, gsel)
        assert np.max(np.abs(o[bi, h] - ro)) < 2e-2, (bi, h)
        assert abs(lse[bi, h] - rl) < 2e-2, (bi, h)


@pytest.mark.parametrize("G,K,d", [(4, 15, 128), (8, 7, 64)])
def test_fused_shared_selection_matches_oracle(G, K, d):
    Hk = 2
    case = inputs.decode_case(80 + G, B=3, Hq=Hk * G, Hk=Hk, d=d, n=2500, b=64, K=K, needles=5,
                              seq_lens=[2500, 1111, 300])
    q, k, v, sl = upload(case)
    mean_k, _, _ = bsa.build_block_summaries(k, 64, sl)
    o, lse, idx, cnt = bsa.decode_step_ex(q, k, v, mean_k, 64, K, bsa.DECODE_SHARED_SELECTION,
                                          seq_lens=sl, append=False)
    torch.cuda.synchronize()
    shared_oracle_check(case, idx.cpu().numpy(), o.float().cpu().numpy(), lse.cpu().numpy())
    exp_cnt = np.minimum(K, (case.seq_lens - 1) // 64)
    assert (cnt.cpu().numpy() == exp_cnt[:, None]).all()


def oracle_bf16_summaries(case):
    """fp64 block means rounded to float32, then to bfloat16: the caller's bf16 mean keys."""
    summ, arr = {}, np.zeros((case.B, case.Hk, -(-case.n // case.b), case.d), np.float32)
    for bi in range(case.B):
        L = int(case.seq_lens[bi])
        for kh in range(case.Hk):
            m = orc.round_bf16(orc.round_f32(orc.block_summaries(case.k[bi, kh, :L], case.b)[0]))
            summ[(bi, kh)] = (m,)
            arr[bi, kh, :m.shape[0]] = m
    return summ, torch.from_numpy(arr).to(DEV, torch.bfloat16)


@pytest.mark.parametrize("shared", [False, True])
def test_fused_bf16_summaries_match_oracle(shared):
    case = inputs.decode_case(85, B=2, Hq=8, Hk=2, d=128, n=3000, b=64, K=9, needles=4,
                              seq_lens=[3000, 1400])
    q, k, v, sl = upload(case)
    summ, mk16 = oracle_bf16_summaries(case)
    flags = bsa.DECODE_BF16_SUMMARIES | (bsa.DECODE_SHARED_SELECTION if shared else 0)
    o, lse, idx, _ = bsa.decode_step_ex(q, k, v, mk16, 64, case.K, flags, seq_lens=sl,
                                        append=False)
    torch.cuda.synchronize()
    idx, o, lse = idx.cpu().numpy(), o.float().cpu().numpy(), lse.cpu().numpy()
    if shared:
        shared_oracle_check(case, idx, o, lse, summaries=summ)
        return
    ref = orc.decode_reference(case.q, case.k, case.v, case.seq_lens, case.b, case.K,
                               summaries=dict(summ))
    for (bi, h), r in ref.items():
        L = int(case.seq_lens[bi])
        sets = orc.valid_selections(r["scores"], orc.sas_num_candidates(L - 1, 64), case.K)
        gsel = sorted(int(x) for x in idx[bi, h] if x >= 0)
        assert sets is not None and gsel in sets, (bi, h, gsel)
        kh = h // 4
        ro, rl = orc.sparse_attention_row(case.q[bi, h], case.k[bi, kh, :L], case.v[bi, kh, :L],
                                          L - 1, 64, gsel)
        assert np.max(np.abs(o[bi, h] - ro)) < 2e-2 and abs(lse[bi, h] - rl) < 2e-2, (bi, h)


def test_fused_bf16_summary_append():
    """The step rewrites the current block's bf16 mean key: bf16 of its float32 mean (within one
    bf16 step of the oracle's rounding of the exact mean)."""
    case = inputs.decode_case(86, B=2, Hq=8, Hk=2, d=128, n=2000, b=64, K=6, needles=3,
                              seq_lens=[2000, 1100])
    q, k, v, sl = upload(case)
    summ, mk16 = oracle_bf16_summaries(case)
    cur = (case.seq_lens - 1) // 64
    for bi in range(2):
        mk16[bi, :, int(cur[bi])] = 99.0
    bsa.decode_step_ex(q, k, v, mk16, 64, 6, bsa.DECODE_BF16_SUMMARIES, seq_lens=sl, append=True)
    torch.cuda.synchronize()
    got = mk16.float().cpu().numpy()
    for bi in range(2):
        for kh in range(2):
            ref = summ[(bi, kh)][0][int(cur[bi])]
            step = np.maximum(np.abs(ref), 1e-30) * 2.0 ** -7
            assert np.all(np.abs(got[bi, kh, int(cur[bi])] - ref) <= step), (bi, kh)


def test_fused_shared_bf16_full_size():
    """The 32K decode workload with both variants: sampled rows against the oracle."""
    case = inputs.decode_case(2000, B=8, Hq=32, Hk=8, d=128, n=32768, b=64, K=15, needles=16,
                              needle_layout="random")
    q, k, v, sl = upload(case)
    mean_k, _, _ = bsa.build_block_summaries(k, 64)
    mk16 = bsa.round_summaries_bf16(mean_k)
    o, lse, idx, _ = bsa.decode_step_ex(q, k, v, mk16, 64, 15,
                                        bsa.DECODE_SHARED_SELECTION | bsa.DECODE_BF16_SUMMARIES,
                                        append=False)
    o2, _, idx2, _ = bsa.decode_step_ex(q, k, v, mean_k, 64, 15, bsa.DECODE_SHARED_SELECTION,
                                        append=False)
    torch.cuda.synchronize()
    # within a group every head holds one selection, and bf16 summaries keep almost all of it
    idx_h = idx.cpu().numpy()
    assert (idx_h.reshape(8, 8, 4, 15) == idx_h.reshape(8, 8, 4, 15)[:, :, :1]).all()
    agree = np.mean([len(set(a) & set(b)) / 15.0 for a, b in
                     zip(idx_h.reshape(-1, 15), idx2.cpu().numpy().reshape(-1, 15))])
    assert agree > 0.9, agree
    rows = [(bi, h) for bi in range(0, 8, 3) for h in range(0, 32, 5)]
    for bi, h in rows:
        L = int(case.seq_lens[bi])
        gsel = sorted(int(x) for x in idx_h[bi, h] if x >= 0)
        ro, rl = orc.sparse_attention_row(case.q[bi, h], case.k[bi, h // 4, :L],
                                          case.v[bi, h // 4, :L], L - 1, 64, gsel)
        assert np.max(np.abs(o[bi, h].float().cpu().numpy() - ro)) < 2e-2, (bi, h)


def test_prepared_decode_step_matches_the_binding_call():
    """bsa.DecodeStep (arguments marshalled once) runs the same step as decode_step_fused."""
    case = inputs.decode_case(87, B=2, Hq=8, Hk=2, d=128, n=2000, b=64, K=6, needles=3,
                              seq_lens=[2000, 1100])
    q, k, v, sl = upload(case)
    mk1, mx1, ce1 = bsa.build_block_summaries(k, 64, sl)
    mk2, mx2, ce2 = mk1.clone(), mx1.clone(), ce1.clone()
    o1, lse1, idx1, cnt1 = bsa.decode_step_fused(q, k, v, mk1, 64, 6, seq_lens=sl, append=True,
                                                 max_norm=mx1, centre=ce1)
    plan = bsa.DecodeStep(q, k, v, mk2, 64, 6, seq_lens=sl, append=True, max_norm=mx2,
                          centre=ce2)
    o2, lse2, idx2, cnt2 = plan()
    o3, _, _, _ = plan(torch.cuda.current_stream())  # a second call reuses the same buffers
    torch.cuda.synchronize()
    assert torch.equal(idx1, idx2) and torch.equal(cnt1, cnt2)
    assert torch.equal(o1, o2) and torch.equal(lse1, lse2) and o3 is o2
    assert torch.equal(mk1, mk2) and torch.equal(mx1, mx2) and torch.equal(ce1, ce2)
