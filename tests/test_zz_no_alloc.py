"""rq_lut_logits_static: the logits call that allocates nothing, for callers
that cannot allocate device memory (memory owned by another runtime's
allocator, serving loops that must not allocate once started).  It must give what
rq_lut_logits gives with a workspace the caller allocated, on consecutive
calls that reuse its fixed scratch, and refuse a call whose workspace would
not fit.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest

from lut_logits_serving_b200 import synth
from tests.parity import RTOL, normwise_err

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import lut_logits_serving_b200 as rq  # noqa: E402


def _call_static(codes, fmt, d, lut, B, cap, logits, argmax):
    return rq.lib().rq_lut_logits_static(
        ctypes.c_void_p(codes.data_ptr()), fmt, d, ctypes.c_void_p(lut.data_ptr()), B,
        ctypes.c_float(cap), ctypes.c_void_p(logits.data_ptr()),
        ctypes.c_void_p(argmax.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("fmt", [0, 2], ids=["u16", "sched"])
def test_static_scratch_matches_the_workspace_call_twice(fmt):
    w = synth.WORKLOADS["g2_b1"]           # needs 24.6 MB of partial sums
    d = rq.dims(w.V, w.D, w.M, w.L, w.K)
    C = torch.from_numpy(synth.codebooks(w.M, w.L, w.K, w.ds, w.sigmas, 0)).cuda()
    c16 = torch.from_numpy(synth.codes(w.V, w.M, w.L, w.K, 1).reshape(w.V, -1)).cuda()
    codes = c16 if fmt == rq.U16 else rq.rq_prepare_sched(c16, d)
    assert rq.rq_logits_workspace_bytes(d, 1, fmt, True) <= (32 << 20)
    for call, seed in enumerate((2, 12)):  # two calls in a row, different tokens
        h = torch.from_numpy(synth.hidden(1, w.D, w.hidden_scale, seed)).cuda()
        lut = rq.rq_lut_build(h, C, d)
        ref, ref_am, _ = rq.rq_lut_logits(codes, fmt, d, lut, 1, w.softcap, want_argmax=True)
        got = torch.full((1, w.V), float("nan"), device="cuda")
        got_am = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        assert _call_static(codes, fmt, d, lut, 1, w.softcap, got, got_am) == 0
        torch.cuda.synchronize()
        err = normwise_err(got.cpu().numpy(), ref.cpu().numpy())
        assert np.all(err <= RTOL), (call, err)
        assert int(got_am.cpu()[0]) == int(ref_am.cpu()[0]), call
    assert rq.rq_device_error() == 0


def test_static_scratch_refuses_what_does_not_fit():
    w = synth.WORKLOADS["g2_b1"]
    d = rq.dims(w.V, w.D, w.M, w.L, w.K)
    assert rq.rq_logits_workspace_bytes(d, 2, rq.U16, True) > (32 << 20)
    codes = torch.zeros((w.V, w.P), dtype=torch.uint16, device="cuda")
    lut = torch.zeros((w.P, w.K, 2), dtype=torch.float32, device="cuda")
    logits = torch.zeros((2, w.V), device="cuda")
    am = torch.zeros((2,), dtype=torch.int32, device="cuda")
    assert _call_static(codes, rq.U16, d, lut, 2, 30.0, logits, am) == 3  # WORKSPACE_TOO_SMALL
    assert torch.count_nonzero(logits).item() == 0                        # nothing launched
