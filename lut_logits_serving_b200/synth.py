"""Seeded synthetic inputs for RQ-LUT logits serving.

This module only draws random numbers in the shapes and distributions of
the workloads; it holds none of the method's arithmetic.  Both the CUDA
library's tests/benchmark and the CPU oracle's tests take their inputs from
here.

Seeds: one ``numpy.random.default_rng`` stream per tensor, derived from a
base seed: codebooks = seed, codes = seed + 1, hidden states = seed + 2,
token ids = seed + 3, rows to encode = seed + 4.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    V: int
    D: int
    M: int
    L: int
    K: int
    B: int                      # tokens per logits call (0: decode-only)
    sigmas: tuple               # codebook std per residual level
    hidden_scale: float         # hidden ~ N(0, 1) * hidden_scale
    softcap: float = 30.0
    packed10: bool = False
    argmax: bool = False
    n_ids: int = 0              # input rows rebuilt per call
    zipf_s: float = 1.1
    decode_scale: float = 0.0   # embedding scale applied to rebuilt rows
    encode: bool = False        # the call encodes V rows instead of scoring them
    topk: int = 0               # > 0: draw the next token from the top-k
    temperature: float = 1.0    # of that draw

    @property
    def ds(self) -> int:
        return self.D // self.M

    @property
    def P(self) -> int:
        return self.M * self.L


# Shapes follow the pages' Gemma-2-2B tied embedding (V=256000, D=2304) with
# the RQ artifact M=384, K=1024, L=2, plus one tiny case for quick checks.
WORKLOADS = {
    "tiny": Workload("tiny", V=4096, D=192, M=32, L=2, K=256, B=1,
                     sigmas=(0.05, 0.01), hidden_scale=1.0),
    "g2_b1": Workload("g2_b1", V=256000, D=2304, M=384, L=2, K=1024, B=1,
                      sigmas=(0.02, 0.005), hidden_scale=40.0 / math.sqrt(2304.0),
                      argmax=True, n_ids=1, decode_scale=math.sqrt(2304.0)),
    # batch 1 on the 10-bit packed artifact (960 bytes per row)
    "g2_b1_packed10": Workload("g2_b1_packed10", V=256000, D=2304, M=384, L=2, K=1024, B=1,
                               sigmas=(0.02, 0.005), hidden_scale=40.0 / math.sqrt(2304.0),
                               packed10=True, argmax=True, n_ids=1,
                               decode_scale=math.sqrt(2304.0)),
    # a batch in the range the L2-served tables take (5 to 16 tokens)
    "g2_b16": Workload("g2_b16", V=256000, D=2304, M=384, L=2, K=1024, B=16,
                       sigmas=(0.02, 0.005), hidden_scale=0.83,
                       argmax=True, n_ids=16, decode_scale=math.sqrt(2304.0)),
    "g2_b32": Workload("g2_b32", V=256000, D=2304, M=384, L=2, K=1024, B=32,
                       sigmas=(0.02, 0.005), hidden_scale=0.83,
                       argmax=True, n_ids=32, decode_scale=math.sqrt(2304.0)),
    "decode512": Workload("decode512", V=256000, D=2304, M=384, L=2, K=1024, B=0,
                          sigmas=(0.02, 0.005), hidden_scale=0.83,
                          n_ids=512, decode_scale=math.sqrt(2304.0)),
    # Generation beyond greedy: the top-50 of the softcapped logits, a draw
    # at temperature 0.8, and the drawn token's input row.
    "g2_b1_topk50": Workload("g2_b1_topk50", V=256000, D=2304, M=384, L=2, K=1024, B=1,
                             sigmas=(0.02, 0.005), hidden_scale=40.0 / math.sqrt(2304.0),
                             topk=50, temperature=0.8, n_ids=1,
                             decode_scale=math.sqrt(2304.0)),
    "packed_b64": Workload("packed_b64", V=256000, D=2304, M=384, L=2, K=1024, B=64,
                           sigmas=(0.02, 0.005), hidden_scale=0.83, packed10=True,
                           argmax=True, n_ids=64, decode_scale=math.sqrt(2304.0)),
    # RQ-compressed MLP weights of a Gemma-2-2B layer, applied without
    # reconstruction (the follow-up the MLP-RQ page names): y = W x with
    # W [out x in], ds = 2, L = 2 and K chosen per matrix for ~10 bits/param
    # including the per-subspace codebooks (L*log2(K)/ds + L*K*32/out):
    # gate/up 8 + 1.8 = 9.8, down 7 + 3.6 = 10.6.
    "mlp_gate_b1": Workload("mlp_gate_b1", V=9216, D=2304, M=1152, L=2, K=256, B=1,
                            sigmas=(0.02, 0.005), hidden_scale=1.0, softcap=0.0),
    "mlp_down_b1": Workload("mlp_down_b1", V=2304, D=9216, M=4608, L=2, K=128, B=1,
                            sigmas=(0.02, 0.005), hidden_scale=1.0, softcap=0.0),
    # Producing the codes: all 256000 embedding rows encoded against the
    # artifact's codebooks (rows ~ N(0, sqrt(0.02^2 + 0.005^2)), the spread of
    # a row the two levels describe).
    "encode_g2": Workload("encode_g2", V=256000, D=2304, M=384, L=2, K=1024, B=0,
                          sigmas=(0.02, 0.005), hidden_scale=0.0, encode=True),
}


def codebooks(M: int, L: int, K: int, ds: int, sigmas, seed: int = 0) -> np.ndarray:
    """float32 [M, L, K, ds]; level l ~ N(0, sigmas[l])."""
    rng = np.random.default_rng(seed)
    C = np.empty((M, L, K, ds), np.float32)
    for l in range(L):
        s = sigmas[min(l, len(sigmas) - 1)]
        C[:, l] = rng.standard_normal((M, K, ds), dtype=np.float32) * np.float32(s)
    return C


def codes(V: int, M: int, L: int, K: int, seed: int = 1) -> np.ndarray:
    """uint16 [V, M, L], uniform in [0, K)."""
    rng = np.random.default_rng(seed)
    return rng.integers(0, K, size=(V, M, L), dtype=np.uint16)


def hidden(B: int, D: int, scale: float, seed: int = 2) -> np.ndarray:
    """float32 [B, D] ~ N(0, 1) * scale."""
    rng = np.random.default_rng(seed)
    return rng.standard_normal((B, D), dtype=np.float32) * np.float32(scale)


def zipf_ids(N: int, V: int, s: float = 1.1, seed: int = 3) -> np.ndarray:
    """int32 [N] token ids: rank r in 1..V drawn with P(r) ~ r^-s by inverse
    CDF on the finite support, mapped through a seeded permutation of
    [0, V) so frequent ids are spread over the vocabulary.  Repeats kept."""
    rng = np.random.default_rng(seed)
    perm = rng.permutation(V)
    w = np.arange(1, V + 1, dtype=np.float64) ** (-s)
    cdf = np.cumsum(w)
    cdf /= cdf[-1]
    u = rng.random(N)
    r = np.minimum(np.searchsorted(cdf, u, side="right"), V - 1)
    return perm[r].astype(np.int32)


def rows(N: int, D: int, sigma: float, seed: int = 4, chunk: int = 16384) -> np.ndarray:
    """float32 [N, D] ~ N(0, sigma), drawn in row chunks of one stream."""
    rng = np.random.default_rng(seed)
    out = np.empty((N, D), np.float32)
    for r0 in range(0, N, chunk):
        r1 = min(N, r0 + chunk)
        out[r0:r1] = rng.standard_normal((r1 - r0, D), dtype=np.float32)
        out[r0:r1] *= np.float32(sigma)
    return out


def row_sigma(w: Workload) -> float:
    """Spread of a row whose levels have std sigmas[l]."""
    return float(math.sqrt(sum(s * s for s in w.sigmas)))


def make(w: Workload, seed: int = 0, V: int | None = None):
    """All inputs of a workload: dict with C, codes, h, ids (V may be cut for
    a smaller sample of the same distributions)."""
    V = w.V if V is None else V
    out = {
        "C": codebooks(w.M, w.L, w.K, w.ds, w.sigmas, seed),
        "codes": codes(V, w.M, w.L, w.K, seed + 1),
    }
    if w.B > 0:
        out["h"] = hidden(w.B, w.D, w.hidden_scale, seed + 2)
    if w.n_ids > 0:
        out["ids"] = zipf_ids(w.n_ids, V, w.zipf_s, seed + 3)
    if w.encode:
        del out["codes"]
        out["X"] = rows(V, w.D, row_sigma(w), seed + 4)
    return out
