"""GPU parity of FS-B ([FreeSolo] "How it differs", FS-B; tree shape of reading R21): the forests
built on the device and the beam search with log-sum-exp re-rank against the fp64 oracle.

A beam search decides at every level which nodes survive, so a near-tie at any cut may send the
device (float32 node scores) and the oracle (float64, rounded to float32) down different valid
paths.  The oracle reports the smallest relative gap at any cut of a query; where it exceeds 1e-4
the selection must be identical, and most queries must be of that kind.  The decode output
(bsa_fsl_decode fed the FS-B selection) is checked against the oracle's two-branch output on the
device's selection."""
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


def _run(seed, B, H, d, n, cell, K, width, positions, bf16=True, lam=0.5):
    fc = inputs.freesolo_case(seed, B=B, H=H, d=d, n=n, cell=cell, K=K, bf16=bf16, lam=lam)
    dt = torch.bfloat16 if bf16 else torch.float32
    k = torch.from_numpy(fc.k).to(DEV, dt)
    v = torch.from_numpy(fc.v).to(DEV, dt)
    pos = np.array(positions, np.int32)
    q_np = np.ascontiguousarray(np.stack([fc.q[bi, :, pos[bi]] for bi in range(B)]))
    q = torch.from_numpy(q_np).to(DEV, dt)
    mean_k, mx, ce = bsa.build_block_summaries(k, cell)
    n_cells = np.array([[orc.freesolo_num_candidates(int(pos[bi]), cell, 128)] * H
                        for bi in range(B)], np.int32)
    forest = bsa.fsb_build(mean_k, mx, ce, torch.from_numpy(n_cells.ravel()).to(DEV))
    lam_t = torch.from_numpy(fc.lam).to(DEV)
    sig_t = torch.from_numpy(fc.sigma).to(DEV)
    pos_t = torch.from_numpy(pos).to(DEV)
    idx, cnt, lse = bsa.fsb_select(q, k, pos_t, cell, forest, lam_t, sig_t, width, K)
    alpha = torch.from_numpy(fc.alpha).to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, idx2, _ = bsa.fsl_decode(q, k, v, pos_t, cell, mean_k, mx, ce, lam_t, sig_t, alpha,
                                idx, cnt, K, window=fc.window, rope_theta=fc.rope_theta,
                                status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(idx, idx2)  # the decode call attends exactly the FS-B cells
    return fc, pos, q_np, n_cells, idx.cpu().numpy(), cnt.cpu().numpy(), lse.cpu().numpy(), \
        o.float().cpu().numpy()


@pytest.mark.parametrize("d,bf16,cell,n,width", [(64, True, 32, 16384, 16), (128, False, 16, 8192, 8),
                                                 (64, True, 64, 32768, 4)])
def test_fsb_select_and_decode_match_oracle(d, bf16, cell, n, width):
    B, H, K = 2, 4, 4
    positions = [n - 1, n // 2 + 300]
    fc, pos, q_np, n_cells, idx, cnt, lse, o = _run(4500 + d + cell, B, H, d, n, cell, K, width,
                                                    positions, bf16)
    checked = 0
    tol = 2e-2 if bf16 else 1e-4
    for bi in range(B):
        i = int(pos[bi])
        for h in range(H):
            summ = orc.block_summaries(fc.k[bi, h].astype(np.float64), cell)
            qv = q_np[bi, h].astype(np.float64)
            lam, sig, al = float(fc.lam[h]), float(fc.sigma[h]), float(fc.alpha[h])
            sel, cand, gap = orc.fsb_select(qv, i, fc.k[bi, h], summ, cell, 128, K, lam, sig,
                                            width)
            got = [int(x) for x in idx[bi, h] if x >= 0]
            assert int(cnt[bi, h]) == len(got) and got == sorted(got)
            if gap > 1e-4:
                checked += 1
                assert got == sel, (bi, h, got, sel, gap)
                want_lse = orc.fsb_rerank_scores(qv, fc.k[bi, h], got, cell)
                assert np.allclose(lse[bi, h, :len(got)], want_lse, rtol=1e-4, atol=1e-4)
            # the output on the device's selection, whatever path it took
            want, _ = orc.freesolo_row(qv, fc.k[bi, h], fc.v[bi, h], i, summ, cell, 128, K,
                                       fc.window, lam, sig, al, fc.rope_theta, selection=got)
            assert float(np.max(np.abs(o[bi, h] - want))) <= tol, (bi, h)
    assert checked >= (B * H) // 2, f"only {checked} of {B * H} queries clear of near-ties"


def test_fsb_beam_covering_every_cell_is_the_exhaustive_rerank():
    """16 candidate cells and a beam of 16: every cell reaches the leaf beam, so the selection is
    the top K of the log-sum-exp re-rank over all of them."""
    B, H, d, n, cell, K, width = 1, 4, 64, 4096, 32, 4, 16
    fc, pos, q_np, n_cells, idx, cnt, lse, o = _run(4600, B, H, d, n, cell, K, width, [600])
    assert (n_cells == 16).all()
    for h in range(H):
        qv = q_np[0, h].astype(np.float64)
        r = orc.round_f32(orc.fsb_rerank_scores(qv, fc.k[0, h], list(range(16)), cell))
        sets = orc.valid_selections(r, 16, K)
        got = [int(x) for x in idx[0, h] if x >= 0]
        assert sets is not None and got in sets, (h, got)


def test_fsb_first_query_block_selects_nothing():
    B, H, d, n, cell, K, width = 1, 2, 64, 2048, 32, 4, 16
    fc, pos, q_np, n_cells, idx, cnt, lse, o = _run(4700, B, H, d, n, cell, K, width, [90])
    assert (cnt == 0).all() and (idx == -1).all()
    for h in range(H):
        summ = orc.block_summaries(fc.k[0, h].astype(np.float64), cell)
        want, _ = orc.freesolo_row(q_np[0, h].astype(np.float64), fc.k[0, h], fc.v[0, h], 90,
                                   summ, cell, 128, K, fc.window, float(fc.lam[h]),
                                   float(fc.sigma[h]), float(fc.alpha[h]), fc.rope_theta)
        assert float(np.max(np.abs(o[0, h] - want))) <= 2e-2
