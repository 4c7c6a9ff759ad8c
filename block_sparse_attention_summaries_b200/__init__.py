"""Python binding of libbsa.so: block-sparse causal attention with per-block summaries (B200).

Every function here only marshals arguments (tensor pointers, sizes, the current CUDA stream) to
the C entry point of the same name in ``include/bsa.h`` (``build_block_summaries`` ->
``bsa_build_block_summaries`` and so on) and allocates output tensors with PyTorch.  All
arithmetic runs in the library's CUDA kernels; there is no CPU or PyTorch fallback: if the shared
library is missing, importing the binding's functions raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbsa.so")

BSA_F32, BSA_BF16 = 0, 1
GATE_NONE, GATE_LOG_SOFTMAX, GATE_OUTER = 0, 1, 2
NORM_SELECTED, NORM_ALL_HISTORY = 0, 1
STATUS_NAMES = {0: "BSA_OK", 1: "BSA_ERR_ARG", 2: "BSA_ERR_SHAPE", 3: "BSA_ERR_DTYPE",
                4: "BSA_ERR_UNSUPPORTED", 5: "BSA_ERR_CUDA", 6: "BSA_ERR_TIMEOUT",
                7: "BSA_ERR_WORKSPACE"}

# (name, restype, argtypes) of every exported entry point, in header order.
_P, _I, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
SIGNATURES = [
    ("bsa_status_string", ctypes.c_char_p, [_I]),
    ("bsa_version", _I, []),
    ("bsa_build_block_summaries", _I, [_P, _I, _I, _I, _I, _I, _I, _P, _I, _I, _P, _P, _P, _P]),
    ("bsa_score_blocks", _I, [_P, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _I, _P, _P,
                              _P]),
    ("bsa_topk_blocks", _I, [_P, _I, _I, _I, _P, _I, _I, _I, _I, _P, _P, _P]),
    ("bsa_decode_step", _I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _I, _P, _P,
                             _I, _I, _P, _P, _P, _P, _P, _P]),
    ("bsa_decode_step_ex", _I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _I, _P,
                                _P, _I, _I, _P, _P, _P, _P, _P, _I, _P]),
    ("bsa_decode_step_ws", _I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _I, _P,
                                _P, _I, _I, _P, _P, _P, _P, _P, _I, _P, _Z, _P]),
    ("bsa_decode_step_workspace_bytes", _Z, [_I, _I, _I, _I, _I, _I, _I, _I, _I]),
    ("bsa_round_summaries_bf16", _I, [_P, _P, ctypes.c_longlong, _P]),
    ("bsa_sparse_attn_fwd", _I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _I, _P, _P, _I,
                                 _I, _I, _P, _I, _P, _P, _P, _Z, _P]),
    ("bsa_sparse_attn_workspace_bytes", _Z, [_I, _I, _I, _I, _I, _I, _I, _I]),
    ("bsa_sparse_attn_decode_noalloc", _I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P,
                                            _I, _I, _I, _P, _I, _P, _P, _P]),
    ("bsa_noalloc_status", _I, [_P]),
    ("bsa_gate_grad_outer", _I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P,
                                 _I, _I, _P, _I, _P, _P]),
    ("bsa_gate_grad", _I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P, _I, _I,
                           _P, _I, _P, _P]),
    ("bsa_selector_grad", _I, [_P, _I, _P, _P, _P, _I, _P, _I, _I, _P, _I, _P]),
    ("bsa_fsl_prune", _I, [_P, _I, _I, _P, _I, _I, _P, _P, _P]),
    ("bsa_fsl_select", _I, [_P, _I, _I, _I, _I, _P, _P, _P, _P, _I, _P, _P, _P, _P, _I, _I, _P,
                            _P, _P]),
    ("bsa_fsl_state_update", _I, [_P, _I, _I, _P, _I, _I, _P, _P, _P, _P, _P, _P]),
    ("bsa_fsl_decode", _I, [_P, _P, _P, _I, _I, _I, _I, _I, _P, _I, _P, _P, _P, _P, _P, _P, _P,
                            _P, _I, _I, _I, ctypes.c_float, _P, _P, _P, _P, _P]),
    ("bsa_fsb_forest_bytes", _Z, [_I, _I, _I, _I]),
    ("bsa_fsb_build", _I, [_P, _P, _P, _I, _I, _I, _I, _P, _P, _Z, _P]),
    ("bsa_fsb_select", _I, [_P, _P, _I, _I, _I, _I, _I, _P, _I, _P, _Z, _P, _P, _I, _I, _P, _P, _P,
                            _P]),
    ("bsa_freesolo_select", _I, [_P, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _I, _P, _P,
                                 _P, _Z, _P]),
    ("bsa_freesolo_select_workspace_bytes", _Z, [_I, _I, _I, _I, _I, _I, _I, _I]),
    ("bsa_freesolo_attn", _I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, ctypes.c_float, _P, _P,
                               _P, _I, _P, _P, _Z, _P]),
    ("bsa_freesolo_workspace_bytes", _Z, [_I, _I, _I, _I, _I, _I, _I]),
    ("bsa_workspace_status", _I, [_P, _P]),
    ("bsa_selftest_bounded_wait", _I, [_P, _I, _P]),
]

_lib = None


class BsaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS_NAMES.get(code, code)}")


def lib() -> ctypes.CDLL:
    """The loaded libbsa.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m block_sparse_attention_summaries_b200.build_lib`")
        h = ctypes.CDLL(LIB_PATH)
        for name, res, args in SIGNATURES:
            fn = getattr(h, name)
            fn.restype = res
            fn.argtypes = args
        _lib = h
    return _lib


def _check(code: int, where: str) -> None:
    if code != 0:
        raise BsaError(code, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device=None):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BSA_BF16
    if t.dtype == torch.float32:
        return BSA_F32
    raise ValueError(f"unsupported dtype {t.dtype}")


def _cuda(*ts):
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise ValueError("tensors must live on a CUDA device")
            if not t.is_contiguous():
                raise ValueError("tensors must be contiguous")


def _host_io(*ts):
    """q / o of a host-I/O decode step: contiguous page-locked host tensors."""
    for t in ts:
        if t is not None:
            if t.is_cuda or not t.is_pinned():
                raise ValueError("host-I/O tensors must be page-locked host memory")
            if not t.is_contiguous():
                raise ValueError("tensors must be contiguous")


def _i32(t):
    if t is None:
        return None
    if t.dtype != torch.int32:
        raise ValueError("index tensors must be int32")
    return t


def _norm_code(norm: str) -> int:
    return {"selected": NORM_SELECTED, "all": NORM_ALL_HISTORY}[norm]


# ---------------------------------------------------------------------------------------------
# Entry points
# ---------------------------------------------------------------------------------------------


def build_block_summaries(k, b, seq_lens=None, first_block=0, num_blocks=-1, mean_k=None,
                          max_norm=None, centre=None):
    """Mean key, max key norm and centre of every block of b tokens of K [B, Hk, n, d]."""
    _cuda(k, seq_lens, mean_k, max_norm, centre)
    B, Hk, n, d = k.shape
    C = (n + b - 1) // b
    if mean_k is None:
        mean_k = torch.empty(B, Hk, C, d, device=k.device, dtype=torch.float32)
    if max_norm is None:
        max_norm = torch.empty(B, Hk, C, device=k.device, dtype=torch.float32)
    if centre is None:
        centre = torch.empty(B, Hk, C, device=k.device, dtype=torch.float32)
    _check(lib().bsa_build_block_summaries(_ptr(k), _dtype_code(k), B, Hk, n, d, b,
                                           _ptr(_i32(seq_lens)), first_block, num_blocks,
                                           _ptr(mean_k), _ptr(max_norm), _ptr(centre),
                                           _stream(k.device)), "bsa_build_block_summaries")
    return mean_k, max_norm, centre


def score_blocks(q, mean_k, n, b, seq_lens=None, max_norm=None, centre=None, lambda_h=None,
                 sigma_h=None, prefix_block=0, scores=None, n_cand=None, Hk=None):
    """Decode block scores [B, Hq, C] of q [B, Hq, d] (and candidate counts [B*Hq])."""
    _cuda(q, mean_k, seq_lens, max_norm, centre, lambda_h, sigma_h, scores, n_cand)
    B, Hq, d = q.shape
    Hk = mean_k.shape[1] if Hk is None else Hk
    C = (n + b - 1) // b
    if scores is None:
        scores = torch.empty(B, Hq, C, device=q.device, dtype=torch.float32)
    if n_cand is None:
        n_cand = torch.empty(B * Hq, device=q.device, dtype=torch.int32)
    _check(lib().bsa_score_blocks(_ptr(q), _dtype_code(q), B, Hq, Hk, n, d, b,
                                  _ptr(_i32(seq_lens)), _ptr(mean_k), _ptr(max_norm),
                                  _ptr(centre), _ptr(lambda_h), _ptr(sigma_h), prefix_block,
                                  _ptr(scores), _ptr(n_cand), _stream(q.device)),
           "bsa_score_blocks")
    return scores, n_cand


def topk_blocks(scores, K, n_cand=None, units=0, q_block=0, b=0, C=None, idx=None, count=None):
    """Top-K block indices (ascending, -1 padded) of every row of scores [..., C]."""
    _cuda(scores, n_cand, idx, count)
    ld = scores.shape[-1]
    C = ld if C is None else C
    rows = scores.numel() // ld
    lead = scores.shape[:-1]
    if idx is None:
        idx = torch.empty(*lead, K, device=scores.device, dtype=torch.int32)
    if count is None:
        count = torch.empty(*lead, device=scores.device, dtype=torch.int32)
    _check(lib().bsa_topk_blocks(_ptr(scores), rows, C, ld, _ptr(_i32(n_cand)), units, q_block, b,
                                 K, _ptr(idx), _ptr(count), _stream(scores.device)),
           "bsa_topk_blocks")
    return idx, count


_workspaces: dict = {}


def workspace(nbytes: int, device) -> torch.Tensor:
    """A zero-filled device workspace of at least ``nbytes`` cached per device (reused)."""
    key = torch.device(device)
    ws = _workspaces.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=key)
        _workspaces[key] = ws
    return ws


def sparse_attn_workspace_bytes(B, Hq, Hk, nq, n, d, b, K) -> int:
    return int(lib().bsa_sparse_attn_workspace_bytes(B, Hq, Hk, nq, n, d, b, K))


def _gate_code(gate):
    """gate: False / None (no gate), True (inner log-gate) or "outer" (gate outside the softmax)."""
    if gate == "outer":
        return GATE_OUTER
    return GATE_LOG_SOFTMAX if gate else GATE_NONE


def sparse_attn_fwd(q, k, v, idx, b, count=None, seq_lens=None, q_block=None, gate=False,
                    norm="selected", scores=None, o=None, lse=None, ws=None):
    """Exact causal softmax over the gathered tokens.

    Decode: q [B, Hq, d] or [B, Hq, 1, d], idx [B, Hq, K].
    Prefill: q [B, Hq, n, d], idx [B, Hq, U, K] with U = ceil(n / q_block).
    Returns (o, lse).
    """
    _cuda(q, k, v, idx, count, seq_lens, scores, o, lse)
    B, Hk, n, d = k.shape
    Hq = q.shape[1]
    decode = q.dim() == 3 or q.shape[2] == 1
    nq = 1 if decode else q.shape[2]
    K = idx.shape[-1]
    if q_block is None:
        q_block = b
    if o is None:
        o = torch.empty(q.shape, device=q.device, dtype=q.dtype)
    if lse is None:
        lse = torch.empty(q.shape[:-1], device=q.device, dtype=torch.float32)
    need = sparse_attn_workspace_bytes(B, Hq, Hk, nq, n, d, b, K)
    if ws is None:
        ws = workspace(need, q.device)
    scores_ld = scores.shape[-1] if scores is not None else 0
    _check(lib().bsa_sparse_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), B, Hq, Hk, nq, n,
                                     d, b, _ptr(_i32(seq_lens)), q_block, _ptr(_i32(idx)),
                                     _ptr(_i32(count)), K,
                                     _gate_code(gate), _norm_code(norm),
                                     _ptr(scores), scores_ld, _ptr(o), _ptr(lse), _ptr(ws),
                                     ws.numel(), _stream(q.device)), "bsa_sparse_attn_fwd")
    return o, lse


def sparse_attn_decode_noalloc(q, k, v, idx, b, count=None, seq_lens=None, gate=False,
                               norm="selected", scores=None, o=None, lse=None):
    """Decode attention like ``sparse_attn_fwd`` but with no workspace: the library's fixed
    per-device scratch array is used instead (for callers that cannot allocate device memory).
    Concurrent calls race on that array; the first call on a device must precede stream
    capture."""
    _cuda(q, k, v, idx, count, seq_lens, scores, o, lse)
    B, Hk, n, d = k.shape
    Hq = q.shape[1]
    K = idx.shape[-1]
    if o is None:
        o = torch.empty(q.shape, device=q.device, dtype=q.dtype)
    if lse is None:
        lse = torch.empty(q.shape[:-1], device=q.device, dtype=torch.float32)
    scores_ld = scores.shape[-1] if scores is not None else 0
    _check(lib().bsa_sparse_attn_decode_noalloc(
        _ptr(q), _ptr(k), _ptr(v), _dtype_code(q), B, Hq, Hk, n, d, b, _ptr(_i32(seq_lens)),
        _ptr(_i32(idx)), _ptr(_i32(count)), K, _gate_code(gate),
        _norm_code(norm), _ptr(scores), scores_ld, _ptr(o), _ptr(lse), _stream(q.device)),
        "bsa_sparse_attn_decode_noalloc")
    return o, lse


def noalloc_status(device=None) -> int:
    """Status of the last allocation-free decode call on ``device`` (0 ok, else
    BSA_ERR_TIMEOUT); reads and clears the status word of the library's fixed array."""
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    with torch.cuda.device(device):  # the array of the current device is read
        return int(lib().bsa_noalloc_status(_stream(torch.device(device))))


def gate_grad(q, k, v, o, lse, dout, idx, b, scores, q_block=None, count=None, norm="selected",
              dg=None, outer=False):
    """dg [B, Hq, U, K] of the inner log-gates (closed form, Eq. 5 of the SAS review), or with
    outer=True of the gates outside the softmax (bsa_gate_grad_outer)."""
    _cuda(q, k, v, o, lse, dout, idx, scores, count, dg)
    B, Hk, n, d = k.shape
    Hq = q.shape[1]
    K = idx.shape[-1]
    if q_block is None:
        q_block = b
    U = (n + q_block - 1) // q_block
    if dg is None:
        dg = torch.empty(B, Hq, U, K, device=q.device, dtype=torch.float32)
    fn = lib().bsa_gate_grad_outer if outer else lib().bsa_gate_grad
    _check(fn(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _dtype_code(q), B, Hq,
              Hk, n, d, b, q_block, _ptr(_i32(idx)), _ptr(_i32(count)), K, _norm_code(norm),
              _ptr(scores), scores.shape[-1], _ptr(dg), _stream(q.device)), "bsa_gate_grad")
    return dg


def selector_grad(scores, n_cand, idx, count, dg, norm, ds=None):
    """ds = dL/ds through the log-softmax gate from dg; leading dims flattened into rows.

    scores [..., C] float32, n_cand [...] int32, idx / dg [..., K], count [...] or None.
    Returns ds [..., C] (0 beyond each row's candidates)."""
    _cuda(scores, n_cand, idx, count, dg, ds)
    C = scores.shape[-1]
    K = idx.shape[-1]
    rows = scores.numel() // C
    if ds is None:
        ds = torch.empty_like(scores)
    _check(lib().bsa_selector_grad(_ptr(scores), C, _ptr(_i32(n_cand)), _ptr(_i32(idx)),
                                   _ptr(None if count is None else _i32(count)), K, _ptr(dg),
                                   int(norm), rows, _ptr(ds), C, _stream(scores.device)),
           "bsa_selector_grad")
    return ds


def fsl_prune(max_norm, n_cells, W, P):
    """FS-L kept cells per row: cand [..., W + P] (ascending, -1 padded), count [...].

    max_norm [..., C] float32; n_cells [...] int32 candidate cells per row."""
    _cuda(max_norm, n_cells)
    C = max_norm.shape[-1]
    rows = max_norm.numel() // C
    lead = max_norm.shape[:-1]
    cand = torch.empty(*lead, W + P, device=max_norm.device, dtype=torch.int32)
    cnt = torch.empty(*lead, device=max_norm.device, dtype=torch.int32)
    _check(lib().bsa_fsl_prune(_ptr(max_norm), rows, C, _ptr(_i32(n_cells)), W, P, _ptr(cand),
                               _ptr(cnt), _stream(max_norm.device)), "bsa_fsl_prune")
    return cand, cnt


class FslState:
    """FS-L fixed-size state of ``rows`` (batch x head) rows: the P kept older cells per row, their
    count and the candidate cells covered (device tensors, zero = empty), plus the kept-cell list
    the last update wrote (bsa_fsl_state_update)."""

    def __init__(self, rows, W, P, device):
        self.W, self.P = W, P
        self.older = torch.full((rows, P), -1, dtype=torch.int32, device=device)
        self.older_count = torch.zeros(rows, dtype=torch.int32, device=device)
        self.state_cells = torch.zeros(rows, dtype=torch.int32, device=device)
        self.cand = torch.full((rows, W + P), -1, dtype=torch.int32, device=device)
        self.cand_count = torch.zeros(rows, dtype=torch.int32, device=device)

    def update(self, max_norm, n_cells):
        """Grow every row's candidate prefix to n_cells [rows] (int32): returns (cand, count)."""
        _cuda(max_norm, n_cells)
        rows = self.older.shape[0]
        C = max_norm.shape[-1]
        _check(lib().bsa_fsl_state_update(_ptr(max_norm), rows, C, _ptr(_i32(n_cells)), self.W,
                                          self.P, _ptr(self.older), _ptr(self.older_count),
                                          _ptr(self.state_cells), _ptr(self.cand),
                                          _ptr(self.cand_count), _stream(max_norm.device)),
               "bsa_fsl_state_update")
        return self.cand, self.cand_count


def fsl_decode(q, k, v, pos, cell, mean_k, max_norm, centre, lambda_h, sigma_h, alpha_h, cand,
               cand_count, K, window=512, rope_theta=10000.0, o=None, idx=None, count=None,
               status=None):
    """FS-L decode output (bsa_fsl_decode): q [B, H, d], k/v [B, H, n, d], pos [B] int32.
    Returns (o, idx, count)."""
    _cuda(q, k, v, pos, mean_k, max_norm, centre, lambda_h, sigma_h, alpha_h, cand, cand_count,
          o, idx, count, status)
    B, H, n, d = k.shape
    if o is None:
        o = torch.empty(B, H, d, device=q.device, dtype=q.dtype)
    if idx is None:
        idx = torch.empty(B, H, K, device=q.device, dtype=torch.int32)
    if count is None:
        count = torch.empty(B, H, device=q.device, dtype=torch.int32)
    _check(lib().bsa_fsl_decode(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), B, H, n, d,
                                _ptr(_i32(pos)), cell, _ptr(mean_k), _ptr(max_norm),
                                _ptr(centre), _ptr(lambda_h), _ptr(sigma_h), _ptr(alpha_h),
                                _ptr(_i32(cand)), _ptr(_i32(cand_count)), cand.shape[-1], K,
                                window, float(rope_theta), _ptr(o), _ptr(idx), _ptr(count),
                                _ptr(status), _stream(q.device)), "bsa_fsl_decode")
    return o, idx, count


def fsb_build(mean_k, max_norm, centre, n_cells, forest=None):
    """Both FS-B forests of every (batch, head) row for its prefix of n_cells [B * H] cells
    (bsa_fsb_build); returns the forest buffer."""
    _cuda(mean_k, max_norm, centre, n_cells, forest)
    B, H, C, d = mean_k.shape
    nbytes = int(lib().bsa_fsb_forest_bytes(B, H, C, d))
    if nbytes == 0:
        raise BsaError(4, "bsa_fsb_forest_bytes")
    if forest is None:
        forest = torch.empty(nbytes, dtype=torch.uint8, device=mean_k.device)
    _check(lib().bsa_fsb_build(_ptr(mean_k), _ptr(max_norm), _ptr(centre), B, H, C, d,
                               _ptr(_i32(n_cells)), _ptr(forest), forest.numel(),
                               _stream(mean_k.device)), "bsa_fsb_build")
    return forest


def fsb_select(q, k, pos, cell, forest, lambda_h, sigma_h, width, K, idx=None, count=None,
               lse=None):
    """FS-B selection of one query per (batch, head) (bsa_fsb_select): q [B, H, d], k [B, H, n, d];
    returns (idx [B, H, K], count [B, H], lse [B, H, K])."""
    _cuda(q, k, pos, forest, lambda_h, sigma_h, idx, count, lse)
    B, H, n, d = k.shape
    if idx is None:
        idx = torch.empty(B, H, K, device=q.device, dtype=torch.int32)
    if count is None:
        count = torch.empty(B, H, device=q.device, dtype=torch.int32)
    if lse is None:
        lse = torch.empty(B, H, K, device=q.device, dtype=torch.float32)
    _check(lib().bsa_fsb_select(_ptr(q), _ptr(k), _dtype_code(q), B, H, n, d, _ptr(_i32(pos)),
                                cell, _ptr(forest), forest.numel(), _ptr(lambda_h),
                                _ptr(sigma_h), width, K, _ptr(idx), _ptr(count), _ptr(lse),
                                _stream(q.device)), "bsa_fsb_select")
    return idx, count, lse


def fsl_select(q, pos, mean_k, max_norm, centre, lambda_h, sigma_h, cand, cand_count, K):
    """FS-L decode selection: idx [B, H, K] (ascending, -1 padded), count [B, H].

    q [B, H, d]; pos [B] int32; summaries [B, H, C, d] / [B, H, C]; lambda_h, sigma_h [H] or
    None; cand / cand_count from fsl_prune."""
    _cuda(q, pos, mean_k, max_norm, centre, lambda_h, sigma_h, cand, cand_count)
    B, H, d = q.shape
    C = mean_k.shape[2]
    idx = torch.empty(B, H, K, device=q.device, dtype=torch.int32)
    cnt = torch.empty(B, H, device=q.device, dtype=torch.int32)
    _check(lib().bsa_fsl_select(_ptr(q), _dtype_code(q), B, H, d, _ptr(_i32(pos)), _ptr(mean_k),
                                _ptr(max_norm), _ptr(centre), C, _ptr(lambda_h), _ptr(sigma_h),
                                _ptr(_i32(cand)), _ptr(_i32(cand_count)), cand.shape[-1], K,
                                _ptr(idx), _ptr(cnt), _stream(q.device)), "bsa_fsl_select")
    return idx, cnt


def freesolo_select(q, mean_k, max_norm, centre, lambda_h, sigma_h, cell, q_block, K,
                    idx=None, count=None, ws=None):
    """Per-query top-K cells of the FreeSolo long branch: idx [B, H, n, K], count [B, H, n].

    ``ws``: a zero-filled uint8 device tensor of at least
    ``bsa_freesolo_select_workspace_bytes`` bytes (allocated here when omitted)."""
    _cuda(q, mean_k, max_norm, centre, lambda_h, sigma_h, idx, count, ws)
    B, H, n, d = q.shape
    if idx is None:
        idx = torch.empty(B, H, n, K, device=q.device, dtype=torch.int32)
    if count is None:
        count = torch.empty(B, H, n, device=q.device, dtype=torch.int32)
    need = int(lib().bsa_freesolo_select_workspace_bytes(_dtype_code(q), B, H, n, d, cell,
                                                         q_block, K))
    if ws is None and need:
        ws = torch.zeros(need, dtype=torch.uint8, device=q.device)
    _check(lib().bsa_freesolo_select(_ptr(q), _dtype_code(q), B, H, n, d, cell, q_block,
                                     _ptr(mean_k), _ptr(max_norm), _ptr(centre), _ptr(lambda_h),
                                     _ptr(sigma_h), K, _ptr(idx), _ptr(count), _ptr(ws),
                                     0 if ws is None else ws.numel(), _stream(q.device)),
           "bsa_freesolo_select")
    return idx, count


def freesolo_attn(q, k, v, alpha_h, idx, count, cell, window, rope_theta=10000.0, o=None,
                  ws=None):
    """FreeSolo two-branch output o [B, H, n, d]."""
    _cuda(q, k, v, alpha_h, idx, count, o)
    B, H, n, d = q.shape
    K = idx.shape[-1]
    if o is None:
        o = torch.empty_like(q)
    need = int(lib().bsa_freesolo_workspace_bytes(_dtype_code(q), B, H, n, d, cell, K))
    if ws is None:
        ws = torch.zeros(need, dtype=torch.uint8, device=q.device)
    _check(lib().bsa_freesolo_attn(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), B, H, n, d, cell,
                                   window, float(rope_theta), _ptr(alpha_h), _ptr(_i32(idx)),
                                   _ptr(_i32(count)), K, _ptr(o), _ptr(ws), ws.numel(),
                                   _stream(q.device)), "bsa_freesolo_attn")
    return o


def workspace_status(ws) -> int:
    """Status word of a workspace (0 ok, else BSA_ERR_TIMEOUT); clears it."""
    return int(lib().bsa_workspace_status(_ptr(ws), _stream(ws.device)))


def selftest_bounded_wait(ws, polls=1000) -> None:
    """Launch the bounded-wait self-test kernel on ``ws`` (see bsa_selftest_bounded_wait)."""
    _check(lib().bsa_selftest_bounded_wait(_ptr(ws), polls, _stream(ws.device)),
           "bsa_selftest_bounded_wait")


def decode_step_fused(q, k, v, mean_k, b, K, seq_lens=None, append=True, max_norm=None,
                      centre=None, lambda_h=None, sigma_h=None, prefix_block=0, o=None, lse=None,
                      idx=None, count=None, status=None):
    """One whole decode step in one launch (bsa_decode_step): returns (o, lse, idx, count)."""
    _cuda(q, k, v, mean_k, seq_lens, max_norm, centre, lambda_h, sigma_h, o, lse, idx, count)
    B, Hk, n, d = k.shape
    Hq = q.shape[1]
    if o is None:
        o = torch.empty(q.shape, device=q.device, dtype=q.dtype)
    if lse is None:
        lse = torch.empty(q.shape[:-1], device=q.device, dtype=torch.float32)
    if idx is None:
        idx = torch.empty(B, Hq, K, device=q.device, dtype=torch.int32)
    if count is None:
        count = torch.empty(B, Hq, device=q.device, dtype=torch.int32)
    _check(lib().bsa_decode_step(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), B, Hq, Hk, n, d, b,
                                 _ptr(_i32(seq_lens)), _ptr(mean_k), _ptr(max_norm), _ptr(centre),
                                 1 if append else 0, _ptr(lambda_h), _ptr(sigma_h), prefix_block,
                                 K, _ptr(o), _ptr(lse), _ptr(idx), _ptr(count), _ptr(status),
                                 _stream(q.device)), "bsa_decode_step")
    return o, lse, idx, count


DECODE_SHARED_SELECTION = 1
DECODE_BF16_SUMMARIES = 2
DECODE_HOST_IO = 4


def decode_step_ex(q, k, v, mean_k, b, K, flags, seq_lens=None, append=True, max_norm=None,
                   centre=None, lambda_h=None, sigma_h=None, prefix_block=0, o=None, lse=None,
                   idx=None, count=None, status=None):
    """bsa_decode_step_ex: the fused decode step with the variants of DECODE_* flags (shared
    selection per kv head; bf16 mean keys).  Returns (o, lse, idx, count)."""
    _cuda(q, k, v, mean_k, seq_lens, max_norm, centre, lambda_h, sigma_h, o, lse, idx, count)
    B, Hk, n, d = k.shape
    Hq = q.shape[1]
    if o is None:
        o = torch.empty(q.shape, device=q.device, dtype=q.dtype)
    if lse is None:
        lse = torch.empty(q.shape[:-1], device=q.device, dtype=torch.float32)
    if idx is None:
        idx = torch.empty(B, Hq, K, device=q.device, dtype=torch.int32)
    if count is None:
        count = torch.empty(B, Hq, device=q.device, dtype=torch.int32)
    _check(lib().bsa_decode_step_ex(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), B, Hq, Hk, n, d, b,
                                    _ptr(_i32(seq_lens)), _ptr(mean_k), _ptr(max_norm),
                                    _ptr(centre), 1 if append else 0, _ptr(lambda_h),
                                    _ptr(sigma_h), prefix_block, K, _ptr(o), _ptr(lse), _ptr(idx),
                                    _ptr(count), _ptr(status), int(flags), _stream(q.device)),
           "bsa_decode_step_ex")
    return o, lse, idx, count


def decode_step_workspace_bytes(B, Hq, Hk, n, d, b, K, flags=0, dtype=None) -> int:
    """Workspace bytes of bsa_decode_step_ws for this shape (0: the step is one launch)."""
    dt = 1 if dtype in (None, torch.bfloat16) else 0
    return int(lib().bsa_decode_step_workspace_bytes(B, Hq, Hk, n, d, b, K, int(flags), dt))


def decode_step_ws(q, k, v, mean_k, b, K, flags=0, ws=None, seq_lens=None, append=True,
                   max_norm=None, centre=None, lambda_h=None, sigma_h=None, prefix_block=0,
                   o=None, lse=None, idx=None, count=None, status=None):
    """bsa_decode_step_ws: the fused decode step; long histories on the 64-token bf16 path run as
    two launches through the workspace ``ws`` (a uint8 device tensor; allocated here when None).
    With DECODE_HOST_IO in ``flags``, q and o are page-locked host tensors (o allocated pinned
    here when None).  Returns (o, lse, idx, count)."""
    host_io = bool(flags & DECODE_HOST_IO)
    if host_io:
        _host_io(q, o)
        _cuda(k, v, mean_k, seq_lens, max_norm, centre, lambda_h, sigma_h, lse, idx, count, ws)
    else:
        _cuda(q, k, v, mean_k, seq_lens, max_norm, centre, lambda_h, sigma_h, o, lse, idx, count,
              ws)
    B, Hk, n, d = k.shape
    Hq = q.shape[1]
    dev = k.device
    if o is None:
        o = (torch.empty(q.shape, dtype=q.dtype, pin_memory=True) if host_io
             else torch.empty(q.shape, device=dev, dtype=q.dtype))
    if lse is None:
        lse = torch.empty(q.shape[:-1], device=dev, dtype=torch.float32)
    if idx is None:
        idx = torch.empty(B, Hq, K, device=dev, dtype=torch.int32)
    if count is None:
        count = torch.empty(B, Hq, device=dev, dtype=torch.int32)
    if ws is None:
        need = decode_step_workspace_bytes(B, Hq, Hk, n, d, b, K, flags, q.dtype)
        ws = torch.empty(max(need, 16), device=dev, dtype=torch.uint8)
    _check(lib().bsa_decode_step_ws(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), B, Hq, Hk, n, d, b,
                                    _ptr(_i32(seq_lens)), _ptr(mean_k), _ptr(max_norm),
                                    _ptr(centre), 1 if append else 0, _ptr(lambda_h),
                                    _ptr(sigma_h), prefix_block, K, _ptr(o), _ptr(lse), _ptr(idx),
                                    _ptr(count), _ptr(status), int(flags), _ptr(ws), ws.numel(),
                                    _stream(dev)), "bsa_decode_step_ws")
    return o, lse, idx, count


class DecodeStep:
    """A prepared bsa_decode_step_ex call for fixed buffers (a serving loop's decode step).

    The argument list (pointers, sizes, flags) is marshalled once here; each call passes it and
    the stream to the C ABI, so a step costs the host one foreign call instead of re-checking and
    re-wrapping every tensor.  The tensors given (and the outputs allocated here) are kept alive
    by this object and must keep their storage: write new queries into ``q`` in place.
    ``outputs`` is (o, lse, idx, count).  With a workspace ``ws`` (a uint8 device tensor of at
    least decode_step_workspace_bytes) the call is bsa_decode_step_ws: long histories take the
    two-launch path, and with DECODE_HOST_IO in ``flags`` q and o are page-locked host tensors
    (the step reads q from and writes o to host memory itself).
    """

    def __init__(self, q, k, v, mean_k, b, K, flags=0, seq_lens=None, append=True,
                 max_norm=None, centre=None, lambda_h=None, sigma_h=None, prefix_block=0,
                 o=None, lse=None, idx=None, count=None, status=None, ws=None):
        host_io = bool(flags & DECODE_HOST_IO)
        if host_io:
            if ws is None:
                raise ValueError("DECODE_HOST_IO needs a workspace")
            _host_io(q, o)
            _cuda(k, v, mean_k, seq_lens, max_norm, centre, lambda_h, sigma_h, lse, idx, count,
                  ws)
        else:
            _cuda(q, k, v, mean_k, seq_lens, max_norm, centre, lambda_h, sigma_h, o, lse, idx,
                  count, ws)
        B, Hk, n, d = k.shape
        Hq = q.shape[1]
        dev = k.device
        if o is None:
            o = (torch.empty(q.shape, dtype=q.dtype, pin_memory=True) if host_io
                 else torch.empty(q.shape, device=dev, dtype=q.dtype))
        if lse is None:
            lse = torch.empty(q.shape[:-1], device=dev, dtype=torch.float32)
        if idx is None:
            idx = torch.empty(B, Hq, K, device=dev, dtype=torch.int32)
        if count is None:
            count = torch.empty(B, Hq, device=dev, dtype=torch.int32)
        sl = _i32(seq_lens)
        self._keep = (q, k, v, mean_k, sl, max_norm, centre, lambda_h, sigma_h, status, ws)
        self.outputs = (o, lse, idx, count)
        self._fn = lib().bsa_decode_step_ex if ws is None else lib().bsa_decode_step_ws
        self._name = "bsa_decode_step_ex" if ws is None else "bsa_decode_step_ws"
        self._args = (_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), B, Hq, Hk, n, d, b, _ptr(sl),
                      _ptr(mean_k), _ptr(max_norm), _ptr(centre), 1 if append else 0,
                      _ptr(lambda_h), _ptr(sigma_h), prefix_block, K, _ptr(o), _ptr(lse),
                      _ptr(idx), _ptr(count), _ptr(status), int(flags))
        if ws is not None:
            self._args = self._args + (_ptr(ws), ws.numel())
        self._device = dev

    def __call__(self, stream=None):
        """Run the step on ``stream`` (a torch.cuda.Stream; default: the current stream)."""
        st = stream if stream is not None else torch.cuda.current_stream(self._device)
        code = self._fn(*self._args, ctypes.c_void_p(st.cuda_stream))
        if code != 0:
            raise BsaError(code, self._name)
        return self.outputs


def round_summaries_bf16(mean_k, out=None):
    """bf16 copy of float32 mean keys (round to nearest even), for DECODE_BF16_SUMMARIES."""
    _cuda(mean_k, out)
    if out is None:
        out = torch.empty(mean_k.shape, device=mean_k.device, dtype=torch.bfloat16)
    _check(lib().bsa_round_summaries_bf16(_ptr(mean_k), _ptr(out), mean_k.numel(),
                                          _stream(mean_k.device)), "bsa_round_summaries_bf16")
    return out


def decode_step(q, k, v, mean_k, b, K, seq_lens=None, append=True, max_norm=None, centre=None,
                out=None):
    """One SAS decode step through the separate calls (the inference algorithm of the SAS review,
    step 6): refresh the summary of the current block, score every history block with
    q . kbar / sqrt(d), take Top-K, attend the selected blocks plus the current block.
    Returns (o, lse, idx)."""
    B, Hk, n, d = k.shape
    if append:
        # first_block = -1: the block holding each row's newest token
        build_block_summaries(k, b, seq_lens, -1, 1, mean_k, max_norm, centre)
    scores, n_cand = score_blocks(q, mean_k, n, b, seq_lens)
    idx, count = topk_blocks(scores, K, n_cand=n_cand)
    o, lse = sparse_attn_fwd(q, k, v, idx, b, count=count, seq_lens=seq_lens, o=out)
    return o, lse, idx
