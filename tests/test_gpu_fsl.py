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
