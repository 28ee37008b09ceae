"""GPU parity of the top-k + temperature-sampling epilogue (rq_topk_sample)
with the oracle.  Both sides see the same fp32 logits: the top-k values and
indices must match exactly (descending, lower index first among equal
values), and the drawn token must be the oracle's (both draw in fp64 from the
same Philox4x64-10 uniform; a disagreement is only possible when u * total
falls within rounding of a running-sum boundary, which the test reports).
Cases span ragged row splits, k from 1 to 1024 (and k = V), ties and
signed zeros, rows whose threshold bin overflows the candidate list (the
exact in-CTA refinement: all-equal rows, values that differ only in low
mantissa bits, a huge tie at the top), and the logits of the full Gemma-2
shaped path."""
import numpy as np
import pytest

import oracle
from lut_logits_serving_b200 import synth
from tests.parity import assert_logits_close

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import lut_logits_serving_b200 as rq  # noqa: E402


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _logits(B, V, seed, coarse=False):
    rng = np.random.default_rng(seed)
    y = rng.normal(0, 3.0, (B, V)).astype(np.float32)
    if coarse:
        y = (np.round(y * 4) / 4).astype(np.float32)   # many exact ties
    return y


def _boundary_margin(val, T, u):
    """Distance of u * total to the nearest running-sum boundary (fp64)."""
    w = np.exp((val.astype(np.float64) - float(val[0])) / T)
    c = np.cumsum(w)
    return float(np.min(np.abs(c - u * c[-1])) / c[-1])


def _check(y, k, T, seed, step):
    gv, gi, gt = rq.rq_topk_sample(dev(y), k, T, seed, step)
    gv, gi, gt = gv.cpu().numpy(), gi.cpu().numpy(), gt.cpu().numpy()
    ov, oi, ot = oracle.sample(y, k, float(np.float32(T)), seed, step)
    assert np.array_equal(gi, oi)
    assert np.array_equal(gv, ov)
    for b in np.nonzero(gt != ot)[0]:
        u = oracle.uniform(seed, step, int(b))
        pytest.fail(f"token row {b}: gpu {gt[b]} oracle {ot[b]}, boundary margin "
                    f"{_boundary_margin(ov[b], float(np.float32(T)), u):.3g}")
    return gt


CASES = [
    # B, V,     k,    coarse
    (1, 5000, 1, False),
    (3, 5000, 7, True),
    (2, 4096, 64, False),
    (4, 70000, 300, True),
    (1, 2049, 1024, False),
    (2, 1024, 1024, False),    # k = V
    (5, 100, 13, True),
    (2, 300000, 1000, False),
]


@pytest.mark.parametrize("B,V,k,coarse", CASES)
@pytest.mark.parametrize("T", [0.7, 1.5])
def test_topk_sample_matches_oracle(B, V, k, coarse, T):
    y = _logits(B, V, seed=V + k, coarse=coarse)
    for step in (0, 1, 12345):
        _check(y, k, T, seed=2024, step=step)


def test_greedy_and_signed_zero():
    y = _logits(3, 9000, 3)
    # temperature 0 and k = 1 are greedy: the first index of the maximum
    for k, T in ((1, 1.0), (40, 0.0), (40, -1.0)):
        _, _, tok = rq.rq_topk_sample(dev(y), k, T, 1, 0)
        assert np.array_equal(tok.cpu().numpy(), np.argmax(y, axis=1))
    # -0 and +0 are equal values: the lower index comes first
    z = np.zeros((1, 3000), np.float32)
    z[0, ::2] = -0.0
    z[0, 2500] = 1.0
    _, gi, _ = rq.rq_topk_sample(dev(z), 5, 1.0, 1, 0)
    assert gi.cpu().numpy().tolist() == [[2500, 0, 1, 2, 3]]


def _heavy_ties(kind, V, seed):
    rng = np.random.default_rng(seed)
    if kind == "all_equal":
        return np.full((2, V), 1.75, np.float32)
    if kind == "low_bits":    # one 12-bit bin: only mantissa bits below it differ
        y = 1.0 + (rng.integers(0, 977, (2, V)) * 2.0 ** -20)
        return y.astype(np.float32)
    y = rng.normal(0, 1, (2, V)).astype(np.float32)    # a huge tie at the top
    y[:, rng.choice(V, 20000, replace=False)] = 9.5
    return y


@pytest.mark.parametrize("kind", ["all_equal", "low_bits", "top_tie"])
@pytest.mark.parametrize("k", [1, 50, 1024])
def test_threshold_bin_overflow(kind, k):
    y = _heavy_ties(kind, 30000, 17)
    for step in (0, 3):
        _check(y, k, 1.1, seed=8, step=step)


def test_many_steps_same_draws():
    y = _logits(1, 20000, 11)
    ov, oi = oracle.topk(y, 20)
    toks = []
    for step in range(300):
        _, _, t = rq.rq_topk_sample(dev(y), 20, 0.9, seed=77, step=step, want_topk=False)
        toks.append(int(t.cpu()[0]))
    want = [int(oi[0, oracle.sample_position(ov[0], float(np.float32(0.9)),
                                             oracle.uniform(77, s, 0))]) for s in range(300)]
    assert toks == want
    assert len(set(toks)) > 5


def test_full_shape_logits():
    """The serving path's own logits (V = 256000, 4 tokens): top-50 and draws
    match the oracle on those logits, and the top-50 set matches the fp64
    reference logits wherever the 50th/51st gap exceeds the logits' bound."""
    w = synth.WORKLOADS["g2_b1"]
    C = synth.codebooks(w.M, w.L, w.K, w.ds, w.sigmas, 0)
    codes = synth.codes(w.V, w.M, w.L, w.K, 1)
    h = synth.hidden(4, w.D, w.hidden_scale, 2)
    d = rq.dims(w.V, w.D, w.M, w.L, w.K)
    logits, _, _ = rq.rq_logits_from_hidden(dev(h), dev(C), dev(codes.reshape(w.V, -1)), rq.U16,
                                            d, w.softcap)
    y = logits.cpu().numpy()
    for step in range(3):
        _check(y, 50, 0.8, seed=5, step=step)
    ref, _ = oracle.reference_logits(codes, C, h, w.softcap)
    assert_logits_close(y, ref)
    _, gi, _ = rq.rq_topk_sample(logits, 50, 0.8, 5, 0)
    gi = gi.cpu().numpy()
    for b in range(4):
        order = np.argsort(-ref[b], kind="stable")
        gap = ref[b, order[49]] - ref[b, order[50]]
        if gap > 1e-5 * np.abs(ref[b]).max():
            assert set(gi[b]) == set(order[:50])
