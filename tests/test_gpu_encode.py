"""GPU parity of the greedy residual encoder (rq_encode) with the oracle's
encoder, bit for bit: every code of small cases that span several row tiles
with a ragged tail, each specialised ds and the generic one, 1 to 3 levels,
codebooks larger than one shared-memory chunk, ties and NaN rows; sampled
rows of the full 256000 x 2304 embedding at the Gemma-2 artifact shape, in
the launch configuration the benchmark times."""
import numpy as np
import pytest

import oracle
from lut_logits_serving_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import lut_logits_serving_b200 as rq  # noqa: E402


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _case(V, D, M, L, K, seed, sigmas=(0.05, 0.01, 0.003)):
    C = synth.codebooks(M, L, K, D // M, sigmas[:L], seed)
    X = synth.rows(V, D, float(np.sqrt(sum(s * s for s in sigmas[:L]))), seed + 4)
    return C, X


def _gpu_encode(X, C):
    M, L, K, ds = C.shape
    d = rq.dims(X.shape[0], X.shape[1], M, L, K)
    out = rq.rq_encode(dev(X), dev(C), d)
    assert rq.rq_device_error() == 0
    return out.cpu().numpy().view(np.uint16).reshape(X.shape[0], M, L)


CASES = [
    # V,    D,   M,  L, K     (ds)
    (3001, 192, 32, 2, 256),    # 6: several 512-row tiles + a ragged tail
    (1, 192, 32, 2, 256),       # a single row
    (517, 64, 32, 2, 37),       # 2, K not a multiple of the unroll
    (700, 128, 32, 1, 64),      # 4, one level
    (600, 96, 12, 3, 100),      # 8, three levels
    (450, 100, 20, 2, 33),      # 5: the generic kernel
    (300, 96, 3, 2, 50),        # 32: the largest generic ds
    (530, 48, 8, 2, 4096),      # 6 with K * ds above one shared-memory chunk
]


@pytest.mark.parametrize("V,D,M,L,K", CASES)
def test_encode_bit_exact(V, D, M, L, K):
    C, X = _case(V, D, M, L, K, seed=V + K)
    got = _gpu_encode(X, C)
    want = oracle.encode(X, C)
    assert np.array_equal(got, want), int((got != want).sum())


def test_encode_ties_nan_and_planted():
    rng = np.random.default_rng(5)
    M, L, K, ds, V = 16, 2, 128, 6, 900
    C = synth.codebooks(M, L, K, ds, (1.0, 1e-3), 5)
    a = rng.integers(0, K, (V, M))
    b = rng.integers(0, K, (V, M))
    X = np.concatenate([(C[m, 0][a[:, m]] + C[m, 1][b[:, m]]).astype(np.float32)
                        for m in range(M)], axis=1)
    C[:, 0, 99] = C[:, 0, 3]                  # duplicate codeword: 3 must win
    X[::7, :ds] = C[0, 0, 3]
    X[5, 2 * ds:3 * ds] = np.nan              # a NaN subspace: code 0 on both levels
    got = _gpu_encode(X, C)
    want = oracle.encode(X, C)
    assert np.array_equal(got, want)
    assert np.all(got[::7, 0, 0] == 3)
    assert got[5, 2, 0] == 0 and got[5, 2, 1] == 0


def test_encode_g2_full_shape_sampled():
    w = synth.WORKLOADS["encode_g2"]
    data = synth.make(w)
    X, C = data["X"], data["C"]
    got = _gpu_encode(X, C)
    rng = np.random.default_rng(13)
    rows = np.unique(np.concatenate([rng.choice(w.V, 192, replace=False),
                                     [0, 1, 511, 512, w.V - 1]]))
    want = oracle.encode(X[rows], C)
    assert np.array_equal(got[rows], want)
    # every code in range, both levels used across the vocabulary
    assert got.max() < w.K
    assert len(np.unique(got[:, 0, 1])) > w.K // 2
