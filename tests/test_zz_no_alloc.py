"""The allocation-free decode entry point, called through the C ABI.

Some callers cannot give the library device memory (an engine with a fixed, pre-planned memory
budget that forbids other allocations; a plugin whose host framework owns the allocator).  For
them bsa_sparse_attn_decode_noalloc runs decode attention on a fixed scratch array inside the
library.  This file checks, on two calls in a row, that its output equals that of the
workspace-taking entry point bsa_sparse_attn_fwd within the bf16 tolerance (2e-2 max abs), with
and without the SAS log-gate, that sampled rows also match the fp64 oracle, that the call through
the Python binding agrees, that the status readback reports no timeout, and that a problem too
large for the fixed array is refused.  It is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import block_sparse_attention_summaries_b200 as bsa
from block_sparse_attention_summaries_b200 import inputs
from oracle import bsa_oracle as orc

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def test_noalloc_decode_matches_workspace_entry_point(bsa_lib):
    case = inputs.decode_case(31, B=4, Hq=16, Hk=4, d=128, n=4096, b=64, K=8, needles=6,
                              seq_lens=[4096, 3000, 65, 1234])
    q = torch.from_numpy(case.q).to(DEV, torch.bfloat16)
    k = torch.from_numpy(case.k).to(DEV, torch.bfloat16)
    v = torch.from_numpy(case.v).to(DEV, torch.bfloat16)
    sl = torch.from_numpy(case.seq_lens).to(DEV)
    mean_k, _, _ = bsa.build_block_summaries(k, case.b, sl)
    scores, n_cand = bsa.score_blocks(q, mean_k, case.n, case.b, sl)
    idx, count = bsa.topk_blocks(scores, case.K, n_cand=n_cand)
    o_ref, lse_ref = bsa.sparse_attn_fwd(q, k, v, idx, case.b, count=count, seq_lens=sl)
    torch.cuda.synchronize()

    # the oracle on sampled rows, evaluated on the GPU's selection (the computed scores may hold
    # near-ties; the selection itself is checked against the oracle elsewhere)
    rows = [(0, 0), (1, 9), (2, 15), (3, 4)]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        o = torch.full_like(o_ref, float("nan"))
        lse = torch.full_like(lse_ref, float("nan"))
        rc = bsa_lib.bsa_sparse_attn_decode_noalloc(
            _p(q), _p(k), _p(v), bsa.BSA_BF16, case.B, case.Hq, case.Hk, case.n, case.d, case.b,
            _p(sl), _p(idx), _p(count), case.K, bsa.GATE_NONE, bsa.NORM_SELECTED, None, 0,
            _p(o), _p(lse), stream)
        assert rc == 0, f"call {call}: status {rc}"
        torch.cuda.synchronize()
        assert bsa.noalloc_status() == 0
        err_o = (o.float() - o_ref.float()).abs().max().item()
        err_l = (lse - lse_ref).abs().max().item()
        assert np.isfinite(err_o) and err_o <= 2e-2, (call, err_o)
        assert np.isfinite(err_l) and err_l <= 2e-2, (call, err_l)
        for bi, h in rows:
            L = int(case.seq_lens[bi])
            sel = sorted(int(x) for x in idx[bi, h].cpu() if x >= 0)
            want_o, want_l = orc.sparse_attention_row(
                case.q[bi, h], case.k[bi, h // (case.Hq // case.Hk), :L],
                case.v[bi, h // (case.Hq // case.Hk), :L], L - 1, case.b, sel)
            assert np.max(np.abs(o[bi, h].float().cpu().numpy() - want_o)) <= 2e-2, (bi, h)
            assert abs(float(lse[bi, h]) - want_l) <= 2e-2, (bi, h)


def test_noalloc_gated_decode_matches_workspace_call_and_oracle(bsa_lib):
    """SAS log-gate (selected normaliser) on supplied selector scores s ~ N(0,1): the gated
    path reads scores and scores_ld; two calls through the C ABI and one through the binding."""
    case = inputs.decode_case(32, B=2, Hq=8, Hk=2, d=64, n=2048, b=64, K=6, needles=0,
                              seq_lens=[2048, 1000], supplied_scores=True)
    q = torch.from_numpy(case.q).to(DEV, torch.bfloat16)
    k = torch.from_numpy(case.k).to(DEV, torch.bfloat16)
    v = torch.from_numpy(case.v).to(DEV, torch.bfloat16)
    sl = torch.from_numpy(case.seq_lens).to(DEV)
    s = torch.from_numpy(case.scores).to(DEV)
    C = s.shape[-1]
    n_cand = torch.from_numpy(np.array([[(int(L) - 1) // case.b] * case.Hq
                                        for L in case.seq_lens], np.int32).ravel()).to(DEV)
    idx, count = bsa.topk_blocks(s, case.K, n_cand=n_cand)
    o_ref, lse_ref = bsa.sparse_attn_fwd(q, k, v, idx, case.b, count=count, seq_lens=sl,
                                         gate=True, norm="selected", scores=s)
    torch.cuda.synchronize()
    rows = [(0, 0), (0, 7), (1, 3), (1, 4)]
    ref = orc.decode_reference(case.q, case.k, case.v, case.seq_lens, case.b, case.K,
                               scores=case.scores, gate_norm="selected", rows=rows)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(3):
        o = torch.full_like(o_ref, float("nan"))
        lse = torch.full_like(lse_ref, float("nan"))
        if call < 2:
            rc = bsa_lib.bsa_sparse_attn_decode_noalloc(
                _p(q), _p(k), _p(v), bsa.BSA_BF16, case.B, case.Hq, case.Hk, case.n, case.d,
                case.b, _p(sl), _p(idx), _p(count), case.K, bsa.GATE_LOG_SOFTMAX,
                bsa.NORM_SELECTED, _p(s), C, _p(o), _p(lse), stream)
            assert rc == 0, f"call {call}: status {rc}"
        else:
            bsa.sparse_attn_decode_noalloc(q, k, v, idx, case.b, count=count, seq_lens=sl,
                                           gate=True, norm="selected", scores=s, o=o, lse=lse)
        torch.cuda.synchronize()
        assert bsa.noalloc_status() == 0
        err_o = (o.float() - o_ref.float()).abs().max().item()
        err_l = (lse - lse_ref).abs().max().item()
        assert np.isfinite(err_o) and err_o <= 2e-2, (call, err_o)
        assert np.isfinite(err_l) and err_l <= 2e-2, (call, err_l)
        for (bi, h), r in ref.items():
            got = sorted(int(x) for x in idx[bi, h].cpu() if x >= 0)
            assert got == r["idx"]
            assert np.max(np.abs(o[bi, h].float().cpu().numpy() - r["o"])) <= 2e-2
            assert abs(float(lse[bi, h]) - r["lse"]) <= 2e-2


def test_noalloc_rejects_problems_beyond_its_scratch(bsa_lib):
    # 4096 sequences x 32 heads of split-K partials need far more than the fixed 4 MiB
    fake = ctypes.c_void_p(0x1000)  # never dereferenced: the size check fails first
    rc = bsa_lib.bsa_sparse_attn_decode_noalloc(
        fake, fake, fake, bsa.BSA_BF16, 4096, 32, 8, 32768, 128, 64, None, fake, None, 15,
        bsa.GATE_NONE, bsa.NORM_SELECTED, None, 0, fake, None, None)
    assert rc == 7  # BSA_ERR_WORKSPACE
