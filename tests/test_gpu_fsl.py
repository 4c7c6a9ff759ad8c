"""GPU parity of FS-L pre-query pruning and selection ([FreeSolo] "How it differs", FS-L)
against the fp64 oracle: pruning bit-exact; selection bit-exact where the K-th and (K+1)-th
kept scores differ by more than 1e-4 relative, else one of the oracle's valid sets."""
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


@pytest.mark.parametrize("C,W,P", [(100, 8, 64), (700, 8, 64), (2048, 8, 64), (5000, 16, 100),
                                   (40, 0, 5)])
def test_fsl_prune_exact(C, W, P):
    rng = np.random.default_rng(C + W)
    rows = 64
    a = (np.round(rng.standard_normal((rows, C)) * 4) / 4).astype(np.float32)  # ties
    a[3, 5] = np.nan
    n_cells = rng.integers(0, C + 1, rows).astype(np.int32)
    n_cells[:4] = [0, 1, min(W + P, C), C]
    cand, cnt = bsa.fsl_prune(torch.from_numpy(a).to(DEV), torch.from_numpy(n_cells).to(DEV), W, P)
    cand, cnt = cand.cpu().numpy(), cnt.cpu().numpy()
    for r in range(rows):
        want = orc.fsl_candidates(a[r].astype(np.float64), int(n_cells[r]), W, P)
        assert cnt[r] == len(want)
        assert list(cand[r, :len(want)]) == want, r
        assert np.all(cand[r, len(want):] == -1)


@pytest.mark.parametrize("lam", [0.5, None])
def test_fsl_select_matches_oracle(lam):
    """FreeSolo decode shapes: 2 batches at different positions of a 64K context, 16 heads."""
    B, H, d, n, cell, K, W, P = 2, 16, 64, 65536, 32, 4, 8, 64
    fc = inputs.freesolo_case(4100, B=B, H=H, d=d, n=n, cell=cell, K=K)
    k = torch.from_numpy(fc.k).to(DEV, torch.bfloat16)
    mean_k, mx, ce = bsa.build_block_summaries(k, cell)
    C = mean_k.shape[2]
    pos = np.array([40000, n - 1], np.int32)
    q_np = np.stack([fc.q[bi, :, pos[bi]] for bi in range(B)])  # [B, H, d]
    q = torch.from_numpy(np.ascontiguousarray(q_np)).to(DEV, torch.bfloat16)
    n_cells = np.array([[orc.freesolo_num_candidates(int(pos[bi]), cell, 128)] * H
                        for bi in range(B)], np.int32)
    cand, ccnt = bsa.fsl_prune(mx, torch.from_numpy(n_cells).to(DEV), W, P)
    lam_t = sig_t = None
    if lam is not None:
        lam_t = torch.full((H,), lam, device=DEV)
        sig_t = torch.full((H,), 4096.0, device=DEV)
    idx, cnt = bsa.fsl_select(q, torch.from_numpy(pos).to(DEV), mean_k, mx, ce, lam_t, sig_t,
                              cand, ccnt, K)
    cand, ccnt, idx, cnt = (x.cpu().numpy() for x in (cand, ccnt, idx, cnt))
    for bi in range(B):
        for h in range(H):
            summ = orc.block_summaries(fc.k[bi, h].astype(np.float64), cell)
            mk, a, c = summ
            nc = int(n_cells[bi, h])
            # the kept set from the oracle's own key norms (fp64 from K, rounded to fp32, the
            # precision the kernel decides in): the W newest cells plus a valid P-set of the older
            # ones -- exact unless the P-th and (P+1)-th norms lie within 1e-4 relative
            recent = list(range(max(0, nc - W), nc))
            older = nc - len(recent)
            p_sets = orc.valid_selections(orc.round_f32(a), older, P)
            assert p_sets is not None
            kept_sets = [sorted(list(ps) + recent) for ps in p_sets]
            assert orc.fsl_candidates(orc.round_f32(a), nc, W, P) in kept_sets
            kept = [int(x) for x in cand[bi, h, :int(ccnt[bi, h])]]
            assert kept in kept_sets, (bi, h)
            assert np.all(cand[bi, h, int(ccnt[bi, h]):] == -1)
            qv = q_np[bi, h].astype(np.float64)
            i = int(pos[bi])
            r = orc.round_f32(orc.freesolo_scores(qv, i, mk, a, c, lam or 0.0, 4096.0, nc))
            sub = r[kept]
            sets = orc.valid_selections(sub, len(kept), K)
            got = [int(x) for x in idx[bi, h] if x >= 0]
            assert cnt[bi, h] == min(K, len(kept))
            assert sets is not None
            assert got in [sorted(kept[j] for j in s) for s in sets], (bi, h, got)


@pytest.mark.parametrize("W,P", [(8, 64), (0, 5), (16, 112), (3, 1)])
def test_fsl_state_update_equals_the_pruning_recomputed(W, P):
    """The fixed-size state grown cell by cell (single cells, jumps of several cells, one large
    first jump) keeps exactly the set bsa_fsl_prune's rule picks from the whole prefix: supplied
    norms with ties and NaN, so bit-exact."""
    rng = np.random.default_rng(100 + W + P)
    rows, C = 40, 2500
    a = (np.round(rng.standard_normal((rows, C)) * 4) / 4).astype(np.float32)
    a[5, 7] = np.nan
    a[6, :50] = np.nan
    a_d = torch.from_numpy(a).to(DEV)
    st = bsa.FslState(rows, W, P, DEV)
    n = np.zeros(rows, np.int64)
    for step in range(12):
        jump = rng.integers(0, 6, rows) if step else rng.integers(0, 1500, rows)
        n = np.minimum(C, n + jump)
        cand, cnt = st.update(a_d, torch.from_numpy(n.astype(np.int32)).to(DEV))
        cand_h, cnt_h = cand.cpu().numpy(), cnt.cpu().numpy()
        for r in range(rows):
            want = orc.fsl_candidates(a[r].astype(np.float64), int(n[r]), W, P)
            assert int(cnt_h[r]) == len(want), (step, r)
            assert list(cand_h[r, :len(want)]) == want, (step, r)
            assert np.all(cand_h[r, len(want):] == -1)
    assert torch.equal(st.state_cells.cpu(), torch.from_numpy(n.astype(np.int32)))


def _fsl_decode_case(seed, B, H, d, n, cell, K, W, P, window, bf16, positions):
    fc = inputs.freesolo_case(seed, B=B, H=H, d=d, n=n, cell=cell, K=K, bf16=bf16)
    dt = torch.bfloat16 if bf16 else torch.float32
    k = torch.from_numpy(fc.k).to(DEV, dt)
    v = torch.from_numpy(fc.v).to(DEV, dt)
    pos = np.array(positions, np.int32)
    q_np = np.ascontiguousarray(np.stack([fc.q[bi, :, pos[bi]] for bi in range(B)]))
    q = torch.from_numpy(q_np).to(DEV, dt)
    mean_k, mx, ce = bsa.build_block_summaries(k, cell)
    st = bsa.FslState(B * H, W, P, DEV)
    n_cells = np.array([[orc.freesolo_num_candidates(int(pos[bi]), cell, 128)] * H
                        for bi in range(B)], np.int32)
    # grow the state over two calls (the prefix of an earlier query, then this one)
    st.update(mx.view(B * H, -1), torch.from_numpy(n_cells.ravel() // 2).to(DEV))
    cand, ccnt = st.update(mx.view(B * H, -1), torch.from_numpy(n_cells.ravel()).to(DEV))
    lam = torch.from_numpy(fc.lam).to(DEV)
    sig = torch.from_numpy(fc.sigma).to(DEV)
    alpha = torch.from_numpy(fc.alpha).to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, idx, cnt = bsa.fsl_decode(q, k, v, torch.from_numpy(pos).to(DEV), cell, mean_k, mx, ce,
                                 lam, sig, alpha, cand.view(B, H, -1), ccnt.view(B, H), K,
                                 window=window, rope_theta=fc.rope_theta, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return fc, pos, q_np, n_cells, cand.view(B, H, -1).cpu().numpy(), ccnt.view(B, H).cpu().numpy(), \
        o.float().cpu().numpy(), idx.cpu().numpy(), cnt.cpu().numpy()


@pytest.mark.parametrize("d,bf16,cell,K,window,n", [(64, True, 32, 4, 512, 65536),
                                                    (128, False, 16, 8, 256, 8192),
                                                    (128, True, 64, 3, 512, 16384)])
def test_fsl_decode_matches_oracle(d, bf16, cell, K, window, n):
    """FS-L decode through the fixed-size state: the kept set checked against the oracle's
    pruning from its own fp64 key norms (valid sets on near-ties), the selection against the
    oracle's over the kept cells (valid sets), and o against the oracle's two-branch FS-L output
    on the GPU's selection (2e-2 bf16, 1e-4 fp32)."""
    B, H, W, P = 2, 4, 8, 64
    positions = [n - 1, n // 2 + 77]
    fc, pos, q_np, n_cells, cand, ccnt, o, idx, cnt = _fsl_decode_case(
        4300 + d + cell, B, H, d, n, cell, K, W, P, window, bf16, positions)
    tol = 2e-2 if bf16 else 1e-4
    for bi in range(B):
        i = int(pos[bi])
        for h in range(H):
            summ = orc.block_summaries(fc.k[bi, h].astype(np.float64), cell)
            mk, a, c = summ
            nc = int(n_cells[bi, h])
            recent = list(range(max(0, nc - W), nc))
            p_sets = orc.valid_selections(orc.round_f32(a), nc - len(recent), P)
            assert p_sets is not None
            kept = [int(x) for x in cand[bi, h, :int(ccnt[bi, h])]]
            assert kept in [sorted(list(ps) + recent) for ps in p_sets], (bi, h)
            qv = q_np[bi, h].astype(np.float64)
            lam, sig, al = float(fc.lam[h]), float(fc.sigma[h]), float(fc.alpha[h])
            r = orc.round_f32(orc.freesolo_scores(qv, i, mk, a, c, lam, sig, nc))
            sets = orc.valid_selections(r[kept], len(kept), K)
            got = [int(x) for x in idx[bi, h] if x >= 0]
            assert int(cnt[bi, h]) == min(K, len(kept))
            assert sets is not None and got in [sorted(kept[j] for j in s) for s in sets], \
                (bi, h, got)
            want, _ = orc.freesolo_row(qv, fc.k[bi, h], fc.v[bi, h], i, summ, cell, 128, K,
                                       window, lam, sig, al, fc.rope_theta, selection=got)
            err = float(np.max(np.abs(o[bi, h] - want)))
            assert err <= tol, (bi, h, err)


def test_fsl_decode_early_query_reads_the_window_only():
    """A query of the first query block has no candidate cell: o is the RoPE window branch alone
    and no cell is selected."""
    B, H, d, n, cell, K, W, P, window = 1, 2, 64, 4096, 32, 4, 8, 64, 512
    fc, pos, q_np, n_cells, cand, ccnt, o, idx, cnt = _fsl_decode_case(
        4400, B, H, d, n, cell, K, W, P, window, True, [100])
    assert (cnt == 0).all() and (idx == -1).all() and (ccnt == 0).all()
    for h in range(H):
        summ = orc.block_summaries(fc.k[0, h].astype(np.float64), cell)
        want, sel = orc.freesolo_row(q_np[0, h].astype(np.float64), fc.k[0, h], fc.v[0, h], 100,
                                     summ, cell, 128, K, window, float(fc.lam[h]),
                                     float(fc.sigma[h]), float(fc.alpha[h]), fc.rope_theta)
        assert sel == []
        assert float(np.max(np.abs(o[0, h] - want))) <= 2e-2
