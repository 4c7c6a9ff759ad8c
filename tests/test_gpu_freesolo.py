"""GPU parity of the FreeSolo two-branch prefill against the fp64 oracle.

Selection: bit-exact cell indices where the oracle's K-th and (K+1)-th scores differ by more than
1e-4 relative, else one of the oracle's valid sets.  Output: max abs error <= 2e-2 (bf16 inputs,
fp32 accumulate), the oracle evaluated with the same valid set.
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


def run_gpu(case):
    q, k, v = (torch.from_numpy(x).to(DEV, torch.bfloat16) for x in (case.q, case.k, case.v))
    lam = torch.from_numpy(case.lam).to(DEV)
    sig = torch.from_numpy(case.sigma).to(DEV)
    alpha = torch.from_numpy(case.alpha).to(DEV)
    mean_k, mx, ce = bsa.build_block_summaries(k, case.cell)
    idx, cnt = bsa.freesolo_select(q, mean_k, mx, ce, lam, sig, case.cell, case.q_block, case.K)
    o = bsa.freesolo_attn(q, k, v, alpha, idx, cnt, case.cell, case.window, case.rope_theta)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), cnt.cpu().numpy(), o.float().cpu().numpy()


def check_rows(case, idx, cnt, o, rows):
    summ = {}
    worst = 0.0
    for (bi, h, i) in rows:
        if (bi, h) not in summ:
            summ[(bi, h)] = orc.block_summaries(case.k[bi, h], case.cell)
        mean_k, max_norm, centre = summ[(bi, h)]
        nc = orc.freesolo_num_candidates(i, case.cell, case.q_block)
        assert cnt[bi, h, i] == min(case.K, nc)
        args = dict(cell=case.cell, q_block=case.q_block, K=case.K, window=case.window,
                    lam=float(case.lam[h]), sigma=float(case.sigma[h]),
                    alpha=float(case.alpha[h]), theta=case.rope_theta)
        gsel = sorted(int(x) for x in idx[bi, h, i] if x >= 0)
        if nc == 0:
            assert gsel == []
            ref, _ = orc.freesolo_row(case.q[bi, h, i], case.k[bi, h], case.v[bi, h], i,
                                      summ[(bi, h)], **args)
        else:
            r = orc.round_f32(orc.freesolo_scores(case.q[bi, h, i], i, mean_k, max_norm, centre,
                                                  args["lam"], args["sigma"], nc))
            sets = orc.valid_selections(r, nc, case.K)
            assert sets is not None and gsel in sets, (bi, h, i, gsel, sets[:2] if sets else None)
            ref, _ = orc.freesolo_row(case.q[bi, h, i], case.k[bi, h], case.v[bi, h], i,
                                      summ[(bi, h)], selection=gsel, **args)
        err = float(np.max(np.abs(o[bi, h, i] - ref)))
        worst = max(worst, err)
        assert err < 2e-2, (bi, h, i, err)
    return worst


@pytest.mark.parametrize("window,sigma", [(100, 300.0), (512, 4096.0)])
def test_freesolo_small(window, sigma):
    case = inputs.freesolo_case(41, B=1, H=2, d=64, n=1000, cell=32, q_block=128, K=4,
                                window=window, sigma=sigma)
    idx, cnt, o = run_gpu(case)
    rng = np.random.default_rng(5)
    rows = [(0, h, i) for h in range(2) for i in
            sorted(set([0, 1, 127, 128, 129, 255, 256, 511, 640, 999]) |
                   set(rng.integers(0, 1000, 30).tolist()))]
    check_rows(case, idx, cnt, o, rows)


def test_freesolo_full_size_sampled():
    """The 64K-token, 16-head FreeSolo workload, checked on sampled queries of three heads."""
    case = inputs.freesolo_case(4000)
    idx, cnt, o = run_gpu(case)
    rng = np.random.default_rng(6)
    rows = []
    for h in (0, 7, 15):
        for i in [0, 127, 128, 4095, 65535] + rng.integers(128, case.n, 8).tolist():
            rows.append((0, h, int(i)))
    check_rows(case, idx, cnt, o, rows)
