"""The allocation-free decode entry point, called through the C ABI.

Some callers cannot give the library device memory (an engine with a fixed, pre-planned memory
budget that forbids other allocations; a plugin whose host framework owns the allocator).  For
them bsa_sparse_attn_decode_noalloc runs decode attention on a fixed scratch array inside the
library.  This file checks, on two calls in a row, that its output equals that of the
workspace-taking entry point bsa_sparse_attn_fwd within the bf16 tolerance (2e-2 max abs), and
that a problem too large for the fixed array is refused.  It is named so that pytest collects it
last.
"""
import ctypes

import numpy as np
import pytest
import torch

import block_sparse_attention_summaries_b200 as bsa
from block_sparse_attention_summaries_b200 import inputs

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
        err_o = (o.float() - o_ref.float()).abs().max().item()
        err_l = (lse - lse_ref).abs().max().item()
        assert np.isfinite(err_o) and err_o <= 2e-2, (call, err_o)
        assert np.isfinite(err_l) and err_l <= 2e-2, (call, err_l)


def test_noalloc_rejects_problems_beyond_its_scratch(bsa_lib):
    # 4096 sequences x 32 heads of split-K partials need far more than the fixed 4 MiB
    fake = ctypes.c_void_p(0x1000)  # never dereferenced: the size check fails first
    rc = bsa_lib.bsa_sparse_attn_decode_noalloc(
        fake, fake, fake, bsa.BSA_BF16, 4096, 32, 8, 32768, 128, 64, None, fake, None, 15,
        bsa.GATE_NONE, bsa.NORM_SELECTED, None, 0, fake, None, None)
    assert rc == 7  # BSA_ERR_WORKSPACE
