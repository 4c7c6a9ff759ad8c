"""Seeded synthetic inputs for block-sparse causal attention.

This module only draws numbers: it holds none of the attention method's arithmetic and is the one
piece of code that both the CUDA path (tests, bench) and the fp64 oracle consume.  Every array is a
NumPy ``float32`` array; for bf16 workloads the values are already rounded to bf16 (round to
nearest even), so ``torch.from_numpy(x).to(torch.bfloat16)`` is exact and the oracle reads the very
same values in fp64.

Streams are counter-based in the sense that every tensor is cut into fixed chunks of ``_CHUNK``
elements and chunk ``j`` of tensor ``name`` is drawn from ``PCG64(SeedSequence([seed, tag(name),
j]))``.  The result therefore does not depend on how many threads draw it, and any slice can be
regenerated alone (``draw_normal(..., rows=...)``).

Workload shapes follow the five configurations the method is measured on (SAS review, "Decoding
efficiency" and "How it works" sections; FreeSolo summary, "How it works" and "Premises and
limits" sections):

* tiny fp32 decode + prefill: B=1, H=2, d=64, n=1024, b=64, K=4, supplied scores s ~ N(0,1);
* SAS-style GQA decode: B=8, Hq=32, Hk=8, d=128, n=32768, b=64, K=15, needles planted;
* long-context decode: B=1, Hq=32, Hk=8, d=128, n=524288, b=64, K=31, 64 strided needles;
* FreeSolo two-branch prefill: B=1, H=16, d=64, n=65536, cells of 32, query block 128, K=4;
* SAS gated training prefill: B=2, Hq=32, Hk=8, d=128, n=16384, b=64, K=16, s and do ~ N(0,1).
"""
from __future__ import annotations

import zlib
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

_CHUNK = 1 << 22  # elements per independently seeded chunk


def _tag(name: str) -> int:
    return zlib.crc32(name.encode()) & 0x7FFFFFFF


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32 holding them."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) & np.uint32(0xFFFF0000)
    return r.view(np.float32)


def draw_normal(seed: int, name: str, shape, bf16: bool, threads: int = 8) -> np.ndarray:
    """N(0,1) float32 array of ``shape`` (bf16-rounded if ``bf16``), chunk-seeded."""
    total = int(np.prod(shape))
    out = np.empty(total, dtype=np.float32)
    nchunks = (total + _CHUNK - 1) // _CHUNK
    tag = _tag(name)

    def fill(j: int) -> None:
        lo, hi = j * _CHUNK, min(total, (j + 1) * _CHUNK)
        g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tag, j])))
        g.standard_normal(hi - lo, dtype=np.float32, out=out[lo:hi])
        if bf16:
            out[lo:hi] = round_bf16(out[lo:hi])

    if nchunks == 1 or threads <= 1:
        for j in range(nchunks):
            fill(j)
    else:
        with ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(fill, range(nchunks)))
    return out.reshape(shape)


def draw_uniform(seed: int, name: str, shape) -> np.ndarray:
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, _tag(name), 0])))
    return g.random(size=shape, dtype=np.float32)


# --------------------------------------------------------------------------------------------
# Workload descriptions
# --------------------------------------------------------------------------------------------


@dataclass
class DecodeCase:
    """One decode step: query at position seq_len-1 of every batch row."""

    B: int
    Hq: int
    Hk: int
    d: int
    n: int
    b: int
    K: int
    bf16: bool
    q: np.ndarray  # [B, Hq, d]
    k: np.ndarray  # [B, Hk, n, d]
    v: np.ndarray  # [B, Hk, n, d]
    seq_lens: np.ndarray  # [B] int32, 1 <= seq_len <= n
    scores: np.ndarray | None = None  # supplied selector scores [B, Hq, C] or None
    needles: dict = field(default_factory=dict)  # (b, kvh) -> planted block indices

    @property
    def C(self) -> int:
        return (self.n + self.b - 1) // self.b


@dataclass
class PrefillCase:
    """Causal self-attention prefill over n positions, selection per query block."""

    B: int
    Hq: int
    Hk: int
    d: int
    n: int
    b: int
    K: int
    q_block: int
    bf16: bool
    q: np.ndarray  # [B, Hq, n, d]
    k: np.ndarray  # [B, Hk, n, d]
    v: np.ndarray  # [B, Hk, n, d]
    scores: np.ndarray | None  # [B, Hq, U, C] selector scores per query block
    dout: np.ndarray | None = None  # [B, Hq, n, d] upstream gradient

    @property
    def C(self) -> int:
        return (self.n + self.b - 1) // self.b

    @property
    def U(self) -> int:
        return (self.n + self.q_block - 1) // self.q_block


@dataclass
class FreeSoloCase:
    B: int
    H: int
    d: int
    n: int
    cell: int
    q_block: int
    K: int
    window: int
    lam: np.ndarray  # [H]
    sigma: np.ndarray  # [H]
    alpha: np.ndarray  # [H]
    rope_theta: float
    q: np.ndarray  # [B, H, n, d]
    k: np.ndarray
    v: np.ndarray


def decode_case(
    seed: int,
    B: int = 8,
    Hq: int = 32,
    Hk: int = 8,
    d: int = 128,
    n: int = 32768,
    b: int = 64,
    K: int = 15,
    needles: int = 16,
    needle_layout: str = "random",
    needle_shift: float = 2.0,
    bf16: bool = True,
    seq_lens=None,
    supplied_scores: bool = False,
) -> DecodeCase:
    """GQA decode inputs with planted needle blocks.

    Keys and values are N(0,1).  For every (batch, kv head) the unit direction u of the sum of the
    group's decode queries is formed and ``needles`` history blocks get ``needle_shift * u`` added
    to every key (a +2 sigma shift along a query direction), either drawn uniformly without
    replacement ("random") or at a uniform stride ("stride").  ``seq_lens`` (optional) makes the
    batch ragged.  ``supplied_scores`` adds selector scores s ~ N(0,1) of shape [B, Hq, C].
    """
    G = Hq // Hk
    q = draw_normal(seed, "q", (B, Hq, d), bf16)
    k = draw_normal(seed, "k", (B, Hk, n, d), bf16)
    v = draw_normal(seed, "v", (B, Hk, n, d), bf16)
    if seq_lens is None:
        seq_lens = np.full(B, n, dtype=np.int32)
    seq_lens = np.asarray(seq_lens, dtype=np.int32)
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, _tag("needles"), 0])))
    planted = {}
    if needles > 0:
        for bi in range(B):
            hist = int(seq_lens[bi] - 1) // b  # number of history blocks of this row
            if hist <= 0:
                continue
            m = min(needles, hist)
            for kh in range(Hk):
                u = q[bi, kh * G:(kh + 1) * G].astype(np.float64).sum(0)
                u /= max(np.linalg.norm(u), 1e-30)
                if needle_layout == "stride":
                    blocks = (np.arange(m) * (hist // m) + (hist // m) // 2).astype(np.int64)
                else:
                    blocks = np.sort(rng.choice(hist, size=m, replace=False))
                shift = (needle_shift * u).astype(np.float32)
                for c in blocks:
                    lo, hi = c * b, min((c + 1) * b, n)
                    blk = k[bi, kh, lo:hi] + shift
                    k[bi, kh, lo:hi] = round_bf16(blk) if bf16 else blk
                planted[(bi, kh)] = blocks
    scores = None
    if supplied_scores:
        scores = draw_normal(seed, "s", (B, Hq, (n + b - 1) // b), False)
    return DecodeCase(B, Hq, Hk, d, n, b, K, bf16, q, k, v, seq_lens, scores, planted)


def tiny_decode_case(seed: int = 1000) -> DecodeCase:
    """Tiny fp32 case: B=1, H=2, d=64, n=1024, b=64, K=4, supplied scores s ~ N(0,1)."""
    return decode_case(seed, B=1, Hq=2, Hk=2, d=64, n=1024, b=64, K=4, needles=0, bf16=False,
                       supplied_scores=True)


def prefill_case(
    seed: int,
    B: int = 2,
    Hq: int = 32,
    Hk: int = 8,
    d: int = 128,
    n: int = 16384,
    b: int = 64,
    K: int = 16,
    q_block: int = 64,
    bf16: bool = True,
    with_dout: bool = True,
    with_scores: bool = True,
) -> PrefillCase:
    """Gated training prefill inputs: Q, K, V, s ~ N(0,1) per (query block, block), do ~ N(0,1)."""
    q = draw_normal(seed, "q", (B, Hq, n, d), bf16)
    k = draw_normal(seed, "k", (B, Hk, n, d), bf16)
    v = draw_normal(seed, "v", (B, Hk, n, d), bf16)
    C = (n + b - 1) // b
    U = (n + q_block - 1) // q_block
    s = draw_normal(seed, "s", (B, Hq, U, C), False) if with_scores else None
    do = draw_normal(seed, "do", (B, Hq, n, d), bf16) if with_dout else None
    return PrefillCase(B, Hq, Hk, d, n, b, K, q_block, bf16, q, k, v, s, do)


def tiny_prefill_case(seed: int = 1000) -> PrefillCase:
    """Tiny fp32 prefill: B=1, H=2, d=64, n=1024, b=64, q_block=64, K=4, s ~ N(0,1)."""
    return prefill_case(seed, B=1, Hq=2, Hk=2, d=64, n=1024, b=64, K=4, q_block=64, bf16=False)


def freesolo_case(
    seed: int,
    B: int = 1,
    H: int = 16,
    d: int = 64,
    n: int = 65536,
    cell: int = 32,
    q_block: int = 128,
    K: int = 4,
    window: int = 512,
    lam: float = 0.5,
    sigma: float = 4096.0,
    rope_theta: float = 10000.0,
    bf16: bool = True,
) -> FreeSoloCase:
    """FreeSolo two-branch prefill inputs: Q, K, V ~ N(0,1), alpha_h ~ U(0,1)."""
    q = draw_normal(seed, "q", (B, H, n, d), bf16)
    k = draw_normal(seed, "k", (B, H, n, d), bf16)
    v = draw_normal(seed, "v", (B, H, n, d), bf16)
    alpha = draw_uniform(seed, "alpha", (H,))
    return FreeSoloCase(B, H, d, n, cell, q_block, K, window,
                        np.full(H, lam, np.float32), np.full(H, sigma, np.float32), alpha,
                        rope_theta, q, k, v)
