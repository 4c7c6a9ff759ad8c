"""The C ABI: the library loads, exports every symbol include/bsa.h declares, and rejects bad
arguments on the host before touching the GPU (CPU only: no compute call is made)."""
import ctypes
import os
import re
import subprocess

import pytest

import block_sparse_attention_summaries_b200 as bsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bsa.h")
FAKE = ctypes.c_void_p(0x1000)  # never dereferenced: every call below fails validation first


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bsa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_hot_path():
    names = declared_functions()
    for must in ["bsa_build_block_summaries", "bsa_score_blocks", "bsa_topk_blocks",
                 "bsa_sparse_attn_fwd", "bsa_gate_grad"]:
        assert must in names


def test_library_exports_every_declared_symbol(bsa_lib):
    for name in declared_functions():
        assert hasattr(bsa_lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", bsa.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r" T (bsa_\w+)", out))
    assert set(declared_functions()) <= exported
    # every binding signature names an exported symbol
    assert {n for n, _, _ in bsa.SIGNATURES} <= exported


def test_binding_covers_header():
    assert {n for n, _, _ in bsa.SIGNATURES} == set(declared_functions())


def test_status_strings(bsa_lib):
    for code in range(8):
        s = bsa_lib.bsa_status_string(code)
        assert s and s != b"unknown status"
    assert bsa_lib.bsa_status_string(42) == b"unknown status"
    assert bsa_lib.bsa_version() >= 100


def test_summaries_rejects_bad_arguments(bsa_lib):
    f = bsa_lib.bsa_build_block_summaries
    ok = dict(k=FAKE, dt=1, B=1, Hk=1, n=128, d=128, b=64, seq=None, first=0, nb=-1,
              mean=FAKE, mx=None, ce=None, st=None)

    def call(**kw):
        a = dict(ok, **kw)
        return f(a["k"], a["dt"], a["B"], a["Hk"], a["n"], a["d"], a["b"], a["seq"], a["first"],
                 a["nb"], a["mean"], a["mx"], a["ce"], a["st"])

    assert call(k=None) == 1
    assert call(mean=None) == 1
    assert call(dt=9) == 3
    assert call(n=0) == 1
    assert call(b=-1) == 1
    assert call(d=96) == 4
    assert call(first=3) == 2  # past the last block
    assert call(first=1, nb=5) == 2
    assert call(first=2, nb=0) == 0  # empty range: nothing to do, nothing launched


def test_score_rejects_bad_arguments(bsa_lib):
    f = bsa_lib.bsa_score_blocks
    base = [FAKE, 1, 2, 8, 2, 1024, 128, 64, None, FAKE, None, None, None, None, 0, FAKE, None,
            None]
    assert f(*base[:0], None, *base[1:]) == 1
    bad = list(base); bad[4] = 3
    assert f(*bad) == 2  # Hq % Hk
    bad = list(base); bad[3] = 24; bad[4] = 2
    assert f(*bad) == 4  # group of 12
    bad = list(base); bad[12] = FAKE  # lambda without sigma
    assert f(*bad) == 1
    bad = list(base); bad[12] = FAKE; bad[13] = FAKE  # lambda without max_norm / centre
    assert f(*bad) == 1
    bad = list(base); bad[6] = 80
    assert f(*bad) == 4


def test_topk_rejects_bad_arguments(bsa_lib):
    f = bsa_lib.bsa_topk_blocks
    assert f(None, 4, 16, 16, None, 0, 0, 0, 4, FAKE, None, None) == 1
    assert f(FAKE, 4, 16, 8, None, 0, 0, 0, 4, FAKE, None, None) == 1  # ld < C
    assert f(FAKE, 4, 16, 16, None, 0, 0, 0, 0, FAKE, None, None) == 1  # K = 0
    assert f(FAKE, 4, 20000, 20000, None, 0, 0, 0, 4, FAKE, None, None) == 4
    assert f(FAKE, 4, 16, 16, None, 0, 0, 0, 300, FAKE, None, None) == 4
    assert f(FAKE, 4, 16, 16, None, 3, 0, 0, 4, FAKE, None, None) == 1  # units w/o q_block
    assert f(FAKE, 0, 16, 16, None, 0, 0, 0, 4, FAKE, None, None) == 0  # no rows: no launch


def test_attention_rejects_bad_arguments(bsa_lib):
    f = bsa_lib.bsa_sparse_attn_fwd
    base = [FAKE, FAKE, FAKE, 1, 2, 8, 2, 1, 1024, 128, 64, None, 64, FAKE, None, 4, 0, 0, None,
            0, FAKE, None, FAKE, 1 << 20, None]
    bad = list(base); bad[1] = None
    assert f(*bad) == 1
    bad = list(base); bad[3] = 5
    assert f(*bad) == 3
    bad = list(base); bad[16] = 1  # gate without scores
    assert f(*bad) == 1
    bad = list(base); bad[16] = 1; bad[18] = FAKE; bad[19] = 3  # scores_ld < C
    assert f(*bad) == 2
    bad = list(base); bad[22] = None  # decode needs a workspace
    assert f(*bad) == 7
    bad = list(base); bad[23] = 16  # too small
    assert f(*bad) == 7
    bad = list(base); bad[7] = 512  # prefill needs nq == n
    assert f(*bad) == 2
    bad = list(base); bad[7] = 1024; bad[11] = FAKE  # prefill takes no seq_lens
    assert f(*bad) == 1
    bad = list(base); bad[10] = 256  # decode block too large
    assert f(*bad) == 4


def test_workspace_size_query(bsa_lib):
    q = bsa_lib.bsa_sparse_attn_workspace_bytes
    n = q(8, 32, 8, 1, 32768, 128, 64, 15)
    assert n > 8 * 32 * (128 + 2) * 4
    assert q(8, 32, 8, 1, 32768, 128, 64, 15) == n  # deterministic, no device query
    assert q(8, 30, 8, 1, 32768, 128, 64, 15) == 0
    assert q(2, 32, 8, 16384, 16384, 128, 64, 16) >= 256


def test_gate_grad_rejects_bad_arguments(bsa_lib):
    f = bsa_lib.bsa_gate_grad
    base = [FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 8, 2, 1024, 128, 64, 64, FAKE, None, 4, 0,
            FAKE, 16, FAKE, None]
    bad = list(base); bad[5] = None
    assert f(*bad) == 1
    bad = list(base); bad[18] = None
    assert f(*bad) == 1
    bad = list(base); bad[19] = 8
    assert f(*bad) == 2
    bad = list(base); bad[17] = 5
    assert f(*bad) == 1


def test_selector_grad_rejects_bad_arguments(bsa_lib):
    f = bsa_lib.bsa_selector_grad
    # scores, scores_ld, n_cand, idx, count, K, dg, norm, rows, ds, ds_ld, stream
    base = [FAKE, 64, FAKE, FAKE, None, 8, FAKE, 1, 100, FAKE, 64, None]
    bad = list(base); bad[0] = None
    assert f(*bad) == 1
    bad = list(base); bad[6] = None
    assert f(*bad) == 1
    bad = list(base); bad[5] = 33
    assert f(*bad) == 4
    bad = list(base); bad[7] = 2
    assert f(*bad) == 1
    bad = list(base); bad[8] = 0
    assert f(*bad) == 1


def test_fsl_rejects_bad_arguments(bsa_lib):
    f = bsa_lib.bsa_fsl_prune
    # max_norm, rows, C, n_cells, W, P, cand, cand_count, stream
    base = [FAKE, 4, 100, FAKE, 8, 64, FAKE, FAKE, None]
    bad = list(base); bad[0] = None
    assert f(*bad) == 1
    bad = list(base); bad[5] = 0
    assert f(*bad) == 1
    bad = list(base); bad[4] = 100
    assert f(*bad) == 4  # W + P > 128
    g = bsa_lib.bsa_fsl_select
    # q, dt, B, H, d, pos, mean_k, max_norm, centre, C, lambda, sigma, cand, cand_count, cand_ld,
    # K, idx, count, stream
    base = [FAKE, 1, 2, 16, 64, FAKE, FAKE, FAKE, FAKE, 2048, FAKE, FAKE, FAKE, FAKE, 72, 4,
            FAKE, None, None]
    bad = list(base); bad[10] = None
    assert g(*bad) == 1  # lambda without sigma
    bad = list(base); bad[14] = 200
    assert g(*bad) == 4
    bad = list(base); bad[4] = 96
    assert g(*bad) == 4


def test_decode_step_ex_rejects_bad_arguments(bsa_lib):
    f = bsa_lib.bsa_decode_step_ex
    base = [FAKE, FAKE, FAKE, 1, 2, 8, 2, 2048, 128, 64, None, FAKE, None, None, 0, None, None, 0,
            15, FAKE, None, None, None, None, 0, None]
    bad = list(base); bad[24] = 4      # unknown flag bit
    assert f(*bad) == 1
    bad = list(base); bad[24] = 2; bad[3] = 0    # bf16 summaries need bf16 K/V
    assert f(*bad) == 4
    bad = list(base); bad[24] = 2; bad[9] = 32   # ... and 64-token blocks
    assert f(*bad) == 4
    bad = list(base); bad[0] = None
    assert f(*bad) == 1
    assert bsa_lib.bsa_round_summaries_bf16(None, FAKE, 16, None) == 1
    assert bsa_lib.bsa_round_summaries_bf16(FAKE, FAKE, -1, None) == 1


def test_outer_gate_arguments(bsa_lib):
    f = bsa_lib.bsa_sparse_attn_fwd
    base = [FAKE, FAKE, FAKE, 1, 2, 8, 2, 1, 1024, 128, 64, None, 64, FAKE, None, 4, 2, 0, FAKE,
            16, FAKE, None, FAKE, 1 << 20, None]
    assert f(*base) == 4                    # decode form: the outer gate is a prefill gate
    bad = list(base); bad[18] = None        # a gate needs scores
    assert f(*bad) == 1
    bad = list(base); bad[16] = 3           # unknown gate mode
    assert f(*bad) == 1
    g = bsa_lib.bsa_gate_grad_outer
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 8, 2, 1024, 128, 64, 64, FAKE, None, 4, 0,
             None, 16, FAKE, None) == 1     # scores missing


def test_decode_step_workspace(bsa_lib):
    """The workspace of bsa_decode_step_ws: none for whole-row histories (<= 512 blocks), other
    dtypes or block sizes; for long histories one record of K keys, K positions, count and
    threshold (padded to 4 words) per chunk and head; a short workspace is refused before any
    launch, and the call without one takes bsa_decode_step_ex's checks."""
    q = bsa_lib.bsa_decode_step_workspace_bytes
    assert q(8, 32, 8, 32768, 128, 64, 15, 0, 1) == 0            # 512 blocks: one launch
    need = q(1, 32, 8, 524288, 128, 64, 31, 0, 1)                # 8192 blocks, 8 groups
    assert need == 8 * 32 * 4 * 64 * 4                           # 32 chunks of 256 blocks
    assert q(1, 32, 8, 524288, 128, 64, 31, 1, 1) == need // 4   # shared selection: one list
    assert q(1, 32, 8, 524288, 128, 64, 31, 0, 0) == 0           # fp32 K/V: one launch
    assert q(1, 32, 8, 524288, 128, 32, 31, 0, 1) == 0           # 32-token blocks: one launch
    assert q(0, 32, 8, 524288, 128, 64, 31, 0, 1) == 0
    f = bsa_lib.bsa_decode_step_ws
    base = [FAKE, FAKE, FAKE, 1, 1, 32, 8, 524288, 128, 64, None, FAKE, None, None, 0, None,
            None, 0, 31, FAKE, None, None, None, None, 0, FAKE, need - 16, None]
    assert f(*base) == 7                                         # BSA_ERR_WORKSPACE
    bad = list(base); bad[25] = ctypes.c_void_p(0x1004)          # misaligned workspace
    assert f(*bad) == 1
    bad = list(base); bad[24] = 8                                # unknown flag bit
    assert f(*bad) == 1
    # host I/O: the workspace also holds the device copy of q, after the chunk lists
    assert q(8, 32, 8, 32768, 128, 64, 15, 4, 1) == 8 * 32 * 128 * 2
    assert q(1, 32, 8, 524288, 128, 64, 31, 4, 1) == need + 32 * 128 * 2
    assert q(1, 32, 8, 524288, 128, 32, 31, 4, 0) == 32 * 128 * 4   # fp32 q, one launch
    short = list(base); short[24] = 4; short[26] = need            # no room for q
    assert f(*short) == 7
    ex = list(base[:25]) + [None]; ex[24] = 4                      # _ex takes no host I/O
    assert bsa_lib.bsa_decode_step_ex(*ex) == 1


def test_freesolo_workspace_size_query(bsa_lib):
    f = bsa_lib.bsa_freesolo_workspace_bytes
    rows = 1 * 16 * 65536
    base = f(1, 1, 16, 65536, 64, 32, 4)             # bf16, cell-major long branch
    assert base >= 256 + 2 * rows * 64 * 2 + rows * 4 * (2 * 64 + 8)
    assert f(1, 1, 16, 65536, 64, 32, 8) > base      # more slots, more partial rows
    assert f(1, 1, 16, 65536, 64, 4, 4) > 0          # other cells: per-unit block unions
    assert f(0, 1, 16, 65536, 64, 32, 4) == 256 + rows * 64 * 4   # fp32: rotated keys only
    assert f(1, 0, 16, 65536, 64, 32, 4) == 0
    assert f(1, 1, 16, 65536, 64, 32, 0) == 0
    assert f(1, 1, 16, 65536, 64, 0, 4) == 0


def test_recorded_traffic_matches_the_kernel_source():
    """The bench reports a kernel's ncu DRAM traffic only while the device code it was captured
    from is unchanged; after a kernel edit the capture must be taken again and re-keyed."""
    import bench
    for (workload, kernel), rec in bench.MEASURED_TRAFFIC.items():
        assert bench.measured_traffic(workload, kernel) == rec["bytes"], (workload, kernel)


def test_recorded_traffic_is_dropped_when_the_device_code_changes(tmp_path, monkeypatch):
    """A record whose source no longer hashes to the captured value reports no traffic (null in
    the bench line), and only the text before the host-code marker counts."""
    import bench
    src = tmp_path / "kernel.cu"
    src.write_text("__global__ void k() {}\nint host_marker() { return 1; }\n")
    h = bench.device_source_hash(str(src), "int host_marker(")
    rec = {"source": str(src), "device_end": "int host_marker(", "sha256_16": h, "bytes": 123}
    monkeypatch.setitem(bench.MEASURED_TRAFFIC, ("w", "k"), rec)
    assert bench.measured_traffic("w", "k") == 123
    src.write_text("__global__ void k() {}\nint host_marker() { return 2; }\n")  # host edit
    assert bench.measured_traffic("w", "k") == 123
    src.write_text("__global__ void k() { int x = 0; }\nint host_marker() { return 2; }\n")
    assert bench.measured_traffic("w", "k") is None
    assert bench.measured_traffic("w", "other") is None
