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


# sigma 300 / 4096: the tensor-core select expands erf about the tile's middle row; sigma 50:
# erf per (query, cell) pair; d = 128: the 128-cell chunk form; q_block 64 / K 8 / fp32 paths too.
@pytest.mark.parametrize("window,sigma,d,q_block,K", [(100, 300.0, 64, 128, 4),
                                                      (512, 4096.0, 64, 128, 4),
                                                      (64, 50.0, 64, 128, 8),
                                                      (256, 1000.0, 128, 128, 3),
                                                      (100, 300.0, 64, 64, 4)])
def test_freesolo_small(window, sigma, d, q_block, K):
    case = inputs.freesolo_case(41, B=1, H=2, d=d, n=1000, cell=32, q_block=q_block, K=K,
                                window=window, sigma=sigma)
    idx, cnt, o = run_gpu(case)
    rng = np.random.default_rng(5)
    rows = [(0, h, i) for h in range(2) for i in
            sorted(set([0, 1, 127, 128, 129, 255, 256, 511, 640, 999]) |
                   set(rng.integers(0, 1000, 30).tolist()))]
    check_rows(case, idx, cnt, o, rows)


@pytest.mark.parametrize("window,d", [(1, 64), (63, 64), (65, 64), (2000, 64), (1, 128),
                                      (65, 128)])
def test_freesolo_window_edges_every_row(window, d):
    """Every row of a ragged case (400 queries: three 128-query tiles and a tail of 16) at the
    window branch's mask edges: the query alone (w = 1), one key less and one more than a 64-key
    block (63, 65), and a window longer than the sequence (no window mask at all)."""
    case = inputs.freesolo_case(49, B=1, H=2, d=d, n=400, cell=32, q_block=128, K=4,
                                window=window, sigma=500.0)
    idx, cnt, o = run_gpu(case)
    check_rows(case, idx, cnt, o, [(0, h, i) for h in range(2) for i in range(case.n)])


@pytest.mark.parametrize("cell,q_block", [(32, 128), (16, 64)])
def test_freesolo_block_count_every_row(cell, q_block):
    """n a multiple of 256, so the long branch places its pairs with the block-aggregated counts
    (shared-memory counters per cell, one global reservation per cell and block): every row of
    two heads."""
    case = inputs.freesolo_case(50, B=1, H=2, d=64, n=1024, cell=cell, q_block=q_block, K=4,
                                window=300, sigma=800.0)
    idx, cnt, o = run_gpu(case)
    check_rows(case, idx, cnt, o, [(0, h, i) for h in range(2) for i in range(case.n)])


@pytest.mark.parametrize("cell", [4, 64])
def test_freesolo_cell_sizes(cell):
    """Cells of 4 keys (per-key masks in the tensor-core long branch) and of 64 (a cell fills a
    block); ragged n."""
    case = inputs.freesolo_case(46, B=1, H=2, d=64, n=1500, cell=cell, q_block=128, K=4,
                                window=200, sigma=600.0)
    idx, cnt, o = run_gpu(case)
    rng = np.random.default_rng(11)
    rows = [(0, h, i) for h in range(2) for i in
            sorted(set([0, 127, 128, 700, 1499]) | set(rng.integers(0, 1500, 12).tolist()))]
    check_rows(case, idx, cnt, o, rows)


@pytest.mark.parametrize("cell", [16, 64])
def test_freesolo_cell_sizes_d128(cell):
    """d = 128 with the smallest and largest cells the cell-major long branch tiles (three and
    two gather stages)."""
    case = inputs.freesolo_case(48, B=1, H=2, d=128, n=1300, cell=cell, q_block=128, K=4,
                                window=150, sigma=700.0)
    idx, cnt, o = run_gpu(case)
    rng = np.random.default_rng(12)
    rows = [(0, h, i) for h in range(2) for i in
            sorted(set([0, 127, 128, 640, 1299]) | set(rng.integers(0, 1300, 12).tolist()))]
    check_rows(case, idx, cnt, o, rows)


def test_freesolo_attn_repeated_and_late_cells():
    """Caller-given slots: a cell repeated within a query's slots counts once, and a cell that
    is not wholly at or before the query is ignored; the long branch uses the rest."""
    case = inputs.freesolo_case(47, B=1, H=2, d=64, n=1024, cell=32, q_block=128, K=4,
                                window=128, sigma=500.0)
    q, k, v = (torch.from_numpy(x).to(DEV, torch.bfloat16) for x in (case.q, case.k, case.v))
    lam = torch.from_numpy(case.lam).to(DEV)
    sig = torch.from_numpy(case.sigma).to(DEV)
    alpha = torch.from_numpy(case.alpha).to(DEV)
    mean_k, mx, ce = bsa.build_block_summaries(k, case.cell)
    idx, cnt = bsa.freesolo_select(q, mean_k, mx, ce, lam, sig, case.cell, case.q_block, case.K)
    rows = [(0, h, i) for h in range(2) for i in (300, 517, 700, 1000)]
    for (bi, h, i) in rows:
        idx[bi, h, i, 1] = idx[bi, h, i, 0]   # repeated
        idx[bi, h, i, 2] = i // case.cell     # the query's own cell: ends after i
    o = bsa.freesolo_attn(q, k, v, alpha, idx, cnt, case.cell, case.window, case.rope_theta)
    torch.cuda.synchronize()
    idx_h, o_h = idx.cpu().numpy(), o.float().cpu().numpy()
    for (bi, h, i) in rows:
        keep = sorted({int(c) for c in idx_h[bi, h, i] if c >= 0 and (c + 1) * case.cell <= i + 1})
        assert len(keep) == 2
        summ = orc.block_summaries(case.k[bi, h], case.cell)
        ref, _ = orc.freesolo_row(case.q[bi, h, i], case.k[bi, h], case.v[bi, h], i, summ,
                                  cell=case.cell, q_block=case.q_block, K=case.K,
                                  window=case.window, lam=float(case.lam[h]),
                                  sigma=float(case.sigma[h]), alpha=float(case.alpha[h]),
                                  theta=case.rope_theta, selection=keep)
        err = float(np.max(np.abs(o_h[bi, h, i] - ref)))
        assert err < 2e-2, (bi, h, i, err)


def test_freesolo_select_two_batches_many_cells():
    """B = 2, 40 cells of 16 per query block: several 256-cell chunks and a ragged last chunk."""
    case = inputs.freesolo_case(43, B=2, H=3, d=64, n=5000, cell=16, q_block=128, K=5,
                                window=128, sigma=2000.0)
    idx, cnt, o = run_gpu(case)
    rng = np.random.default_rng(9)
    rows = [(int(b), int(h), int(i)) for b, h, i in
            zip(rng.integers(0, 2, 24), rng.integers(0, 3, 24), rng.integers(0, 5000, 24))]
    rows += [(1, 2, 4999), (0, 0, 4096), (1, 1, 4224)]
    check_rows(case, idx, cnt, o, rows)


def test_freesolo_select_status_clean():
    case = inputs.freesolo_case(44, B=1, H=2, d=64, n=2048, cell=32, q_block=128, K=4)
    q = torch.from_numpy(case.q).to(DEV, torch.bfloat16)
    k = torch.from_numpy(case.k).to(DEV, torch.bfloat16)
    lam = torch.from_numpy(case.lam).to(DEV)
    sig = torch.from_numpy(case.sigma).to(DEV)
    mean_k, mx, ce = bsa.build_block_summaries(k, case.cell)
    need = int(bsa.lib().bsa_freesolo_select_workspace_bytes(bsa.BSA_BF16, 1, 2, 2048, 64, 32,
                                                             128, 4))
    assert need > 0
    ws = torch.zeros(need, dtype=torch.uint8, device=DEV)
    bsa.freesolo_select(q, mean_k, mx, ce, lam, sig, case.cell, case.q_block, case.K, ws=ws)
    assert bsa.workspace_status(ws) == 0
    with pytest.raises(RuntimeError):
        bsa.freesolo_select(q, mean_k, mx, ce, lam, sig, case.cell, case.q_block, case.K,
                            ws=ws[:need - 1])


def test_freesolo_attn_status_clean():
    """The tensor-core window and long branches leave the workspace status word at zero."""
    case = inputs.freesolo_case(45, B=1, H=2, d=64, n=3000, cell=32, q_block=128, K=4,
                                window=256, sigma=1000.0)
    q, k, v = (torch.from_numpy(x).to(DEV, torch.bfloat16) for x in (case.q, case.k, case.v))
    lam = torch.from_numpy(case.lam).to(DEV)
    sig = torch.from_numpy(case.sigma).to(DEV)
    alpha = torch.from_numpy(case.alpha).to(DEV)
    mean_k, mx, ce = bsa.build_block_summaries(k, case.cell)
    idx, cnt = bsa.freesolo_select(q, mean_k, mx, ce, lam, sig, case.cell, case.q_block, case.K)
    need = int(bsa.lib().bsa_freesolo_workspace_bytes(bsa.BSA_BF16, 1, 2, 3000, 64,
                                                         case.cell, case.K))
    ws = torch.zeros(need, dtype=torch.uint8, device=DEV)
    bsa.freesolo_attn(q, k, v, alpha, idx, cnt, case.cell, case.window, case.rope_theta, ws=ws)
    assert bsa.workspace_status(ws) == 0


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
