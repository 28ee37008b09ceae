"""The greedy pick over a vocabulary split across ranks: every shard runs the
fused call on its own code rows, its per-token winner is exchanged, and the
merge must give exactly the unsharded argmax (rows are independent, so a
shard's logits are bit-identical to the same rows of the full run).  The ranks
are run one after another on one GPU; the exchange is the stacking that an
all-gather produces."""
import numpy as np
import pytest

import oracle
from lut_logits_serving_b200 import synth
from tests.parity import check_argmax

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import lut_logits_serving_b200 as rq  # noqa: E402


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def make_case(V, M, K, B, seed):
    D = 6 * M
    C = synth.codebooks(M, 2, K, 6, (0.05, 0.01), seed)
    codes = synth.codes(V, M, 2, K, seed + 1)
    h = synth.hidden(B, D, 1.0, seed + 2)
    return C, codes, h


def sharded(C, codes, h, world, cap=30.0):
    """Logits per shard and the merged pick, ranks run in turn."""
    V, M = codes.shape[0], codes.shape[1]
    K = C.shape[2]
    dC, dh = dev(C), dev(h)
    vals, idxs, parts = [], [], []
    for rank in range(world):
        r0, r1 = rq.shard_rows(V, rank, world)
        d = rq.dims(r1 - r0, 6 * M, M, 2, K)
        logits, am, _ = rq.rq_logits_from_hidden(dh, dC, dev(codes[r0:r1].reshape(r1 - r0, -1)),
                                                 rq.U16, d, cap, want_argmax=True)
        val, gidx = rq.rq_argmax_candidates(logits, am, r0)
        vals.append(val)
        idxs.append(gidx)
        parts.append(logits)
    pick = rq.rq_argmax_merge(torch.stack(vals), torch.stack(idxs))
    return torch.cat(parts, dim=1), pick


@pytest.mark.parametrize("B", [1, 8, 40])
@pytest.mark.parametrize("world", [2, 3, 8])
def test_sharded_pick_equals_the_full_run(B, world):
    V, M, K = 6007, 16, 256
    C, codes, h = make_case(V, M, K, B, seed=B + world)
    d = rq.dims(V, 6 * M, M, 2, K)
    full, am, _ = rq.rq_logits_from_hidden(dev(h), dev(C), dev(codes.reshape(V, -1)), rq.U16, d,
                                           30.0, want_argmax=True)
    parts, pick = sharded(C, codes, h, world)
    assert torch.equal(parts, full)
    assert torch.equal(pick, am)
    T = oracle.lut_build(h, C, "f64")
    check_argmax(pick.cpu().numpy(), oracle.softcap(oracle.logits_lut(codes, T), 30.0))
    assert rq.rq_device_error() == 0


def test_ties_across_shards_go_to_the_lowest_row():
    """A copy of the winning row in an earlier shard has the same logit; the
    merged pick is the copy (lower global index), as in the unsharded argmax."""
    V, M, K, B = 3000, 8, 128, 1
    C, codes, h = make_case(V, M, K, B, seed=5)
    d = rq.dims(V, 6 * M, M, 2, K)
    _, am, _ = rq.rq_logits_from_hidden(dev(h), dev(C), dev(codes.reshape(V, -1)), rq.U16, d,
                                        30.0, want_argmax=True)
    win = int(am[0])
    twin = 7 if win > 1500 else 2990          # in another shard of two
    codes[twin] = codes[win]
    _, am2, _ = rq.rq_logits_from_hidden(dev(h), dev(C), dev(codes.reshape(V, -1)), rq.U16, d,
                                         30.0, want_argmax=True)
    _, pick = sharded(C, codes, h, 2)
    assert int(am2[0]) == min(win, twin)
    assert int(pick[0]) == min(win, twin)


def test_merge_orders_nan_and_ties():
    """The merge's order: larger value, then lower index; NaN never wins."""
    nan = float("nan")
    val = torch.tensor([[1.0, nan, 2.0, 5.0], [1.0, 3.0, nan, 5.0], [0.5, 3.0, 2.0, nan]],
                       device="cuda")
    idx = torch.tensor([[10, 1, 7, 9], [4, 8, 2, 3], [1, 5, 6, 0]], dtype=torch.int32,
                       device="cuda")
    out = rq.rq_argmax_merge(val, idx)
    assert out.cpu().tolist() == [4, 5, 6, 3]


def test_sharded_logits_on_one_rank():
    """rq_sharded_logits without a process group is the unsharded call."""
    V, M, K, B = 2048, 8, 256, 4
    C, codes, h = make_case(V, M, K, B, seed=9)
    d = rq.dims(V, 6 * M, M, 2, K)
    args = (dev(h), dev(C), dev(codes.reshape(V, -1)), rq.U16, d)
    logits, pick, _ = rq.rq_sharded_logits(*args, 0, 30.0)
    full, am, _ = rq.rq_logits_from_hidden(*args, 30.0, want_argmax=True)
    assert torch.equal(logits, full) and torch.equal(pick, am)
