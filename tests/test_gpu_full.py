"""GPU parity at the full Gemma-2 shapes (V=256000, D=2304, M=384, L=2,
K=1024), in the launch configuration the benchmark times.

* decode batch 1, uint16, bank-scheduled and 10-bit packed codes: all
  256000 logits and the argmax against the oracle (the oracle does the full
  row sweep in about a second);
* batch 32, uint16 codes, one code pass for all tokens: all 32 x 256000
  logits and every token's argmax, on every kernel choice, and on the
  bank-scheduled layout;
* batch 64, 10-bit packed codes, fused build + unpack + sum + softcap +
  argmax: all 64 x 256000 logits and every token's argmax;
* 512 Zipf-drawn input rows rebuilt in bf16: all of them, bit for bit.
"""
import numpy as np
import pytest

import oracle
from lut_logits_serving_b200 import synth
from tests.parity import assert_logits_close, check_argmax

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import lut_logits_serving_b200 as rq  # noqa: E402


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


@pytest.fixture(scope="module")
def g2():
    w = synth.WORKLOADS["g2_b1"]
    C = synth.codebooks(w.M, w.L, w.K, w.ds, w.sigmas, 0)
    codes = synth.codes(w.V, w.M, w.L, w.K, 1)
    d = rq.dims(w.V, w.D, w.M, w.L, w.K)
    dc = dev(codes.reshape(w.V, -1))
    return dict(C=C, codes=codes, d=d, dC=dev(C), dc=dc)


def _sample_rows(V, n, seed):
    rng = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([rng.choice(V, n, replace=False), [0, V - 1]]))
    return rows.astype(np.int64)


def test_g2_batch1_full_sweep(g2):
    w = synth.WORKLOADS["g2_b1"]
    h = synth.hidden(1, w.D, w.hidden_scale, 2)
    d = g2["d"]
    lut = rq.rq_lut_build(dev(h), g2["dC"], d)
    logits, am, _ = rq.rq_lut_logits(g2["dc"], rq.U16, d, lut, 1, w.softcap, want_argmax=True)
    got = logits.cpu().numpy()
    T = oracle.lut_build(h, g2["C"], "f64")
    ref = oracle.softcap(oracle.logits_lut(g2["codes"], T), w.softcap)
    err = assert_logits_close(got, ref)
    print(f"g2_b1 normwise error {err:.3g}")
    assert check_argmax(am.cpu().numpy(), ref) == 0
    # the step the benchmark times: fused call, argmax only
    _, am2, _ = rq.rq_logits_from_hidden(dev(h), g2["dC"], g2["dc"], rq.U16, d, w.softcap,
                                         want_logits=False, want_argmax=True)
    assert int(am2.cpu()[0]) == int(am.cpu()[0])
    # the bank-scheduled layout: same logits up to summation order
    sched = rq.rq_prepare_sched(g2["dc"], d)
    logits3, am3, _ = rq.rq_logits_from_hidden(dev(h), g2["dC"], sched, rq.SCHED, d, w.softcap,
                                               want_argmax=True)
    err3 = assert_logits_close(logits3.cpu().numpy(), ref)
    print(f"g2_b1 sched normwise error {err3:.3g}")
    assert check_argmax(am3.cpu().numpy(), ref) == 0
    # the benchmark's step: logits, argmax and the picked token's input row
    logits4, am4, rows4, _ = rq.rq_greedy_step(dev(h), g2["dC"], sched, rq.SCHED, d, w.softcap,
                                               scale=w.decode_scale)
    assert torch.equal(am4, am3)
    assert_logits_close(logits4.cpu().numpy(), ref)
    want = oracle.decode_rows_bf16(am4.cpu().numpy().astype(np.int32), g2["codes"], g2["C"],
                                   w.decode_scale)
    assert np.array_equal(rows4.view(torch.int16).cpu().numpy().view(np.uint16), want)
    # 10-bit packed codes: the same pass over 48-byte windows of the packed rows
    packed = rq.rq_pack10(g2["dc"], d)
    out5 = torch.full((1, w.V), float("nan"), device="cuda")
    logits5, am5, rows5, _ = rq.rq_greedy_step(dev(h), g2["dC"], packed, rq.PACKED10, d,
                                               w.softcap, scale=w.decode_scale, logits=out5)
    err5 = assert_logits_close(logits5.cpu().numpy(), ref)
    print(f"g2_b1 packed10 normwise error {err5:.3g}")
    assert check_argmax(am5.cpu().numpy(), ref) == 0
    assert torch.equal(am5, am3)
    assert torch.equal(rows5, rows4)
    # the rotated 10-bit layout: the same sums in another order
    rot, (steps, passes) = rq.rq_prepare_rot10(g2["dc"], d, stats=True)
    print(f"g2_b1 rotated slices: {passes / steps:.3f} bank passes per step")
    logits6, am6, rows6, _ = rq.rq_greedy_step(dev(h), g2["dC"], rot, rq.ROT10, d, w.softcap,
                                               scale=w.decode_scale)
    err6 = assert_logits_close(logits6.cpu().numpy(), ref)
    print(f"g2_b1 rot10 normwise error {err6:.3g}")
    assert check_argmax(am6.cpu().numpy(), ref) == 0
    assert torch.equal(am6, am3)
    assert torch.equal(rows6, rows4)
    assert rq.rq_device_error() == 0


_REF = {}


def _full_ref(g2, w):
    """The oracle's fp64 logits of every token and row (computed once per
    workload; the oracle's row loop runs on all host cores)."""
    if w.name not in _REF:
        h = synth.hidden(w.B, w.D, w.hidden_scale, 2)
        T = oracle.lut_build(h, g2["C"], "f64")
        _REF[w.name] = (h, oracle.softcap(oracle.logits_lut(g2["codes"], T), w.softcap))
    return _REF[w.name]


def elementwise_rel(got, ref, floor=1e-2):
    """Largest elementwise relative error over the logits whose magnitude is
    at least `floor` of their token's largest (reported, not gated: below that
    the ratio measures cancellation, not the kernel)."""
    ref = np.asarray(ref, np.float64)
    big = np.abs(ref) >= floor * np.max(np.abs(ref), axis=1, keepdims=True)
    return float(np.max(np.abs(got.astype(np.float64)[big] - ref[big]) / np.abs(ref[big])))


def _batched(g2, w, fmt, path=None):
    d = g2["d"]
    h, ref = _full_ref(g2, w)
    codes_dev = (g2["dc"] if fmt == rq.U16 else
                 rq.rq_prepare_sched(g2["dc"], d) if fmt == rq.SCHED else
                 rq.rq_pack10(g2["dc"], d))
    # NaN-filled output: a kernel that writes nothing cannot pass on stale memory
    out = torch.full((w.B, w.V), float("nan"), device="cuda")
    logits, am, _ = rq.rq_logits_from_hidden(dev(h), g2["dC"], codes_dev, fmt, d, w.softcap,
                                             want_argmax=True, logits=out, path=path)
    assert rq.rq_device_error() == 0
    got = logits.cpu().numpy()
    amv = am.cpu().numpy()
    err = assert_logits_close(got, ref)          # every token, every row
    ties = check_argmax(amv, ref)                 # every token
    # every token's argmax is also the argmax of the GPU's own logits
    assert np.array_equal(amv, np.argmax(got, axis=1))
    return err, elementwise_rel(got, ref), ties


@pytest.mark.parametrize("path", [None, rq.PATH_TABLES, rq.PATH_DECODE_FP32, rq.PATH_DECODE_TC])
def test_g2_batch32_one_code_pass(g2, path):
    w = synth.WORKLOADS["g2_b32"]
    err, rel, ties = _batched(g2, w, rq.U16, path)
    print(f"g2_b32 path {path} normwise error {err:.3g}, elementwise relative error "
          f"(|ref| >= 1e-2 max) {rel:.3g}, ties {ties}")
    assert ties == 0
    assert rq.rq_device_error() == 0


def test_g2_batch32_scheduled_codes(g2):
    """The batch-1 layout also serves a 32-token group: the tensor-core decode
    puts its slices back in pair order."""
    w = synth.WORKLOADS["g2_b32"]
    err, rel, ties = _batched(g2, w, rq.SCHED)
    print(f"g2_b32 scheduled codes normwise error {err:.3g}, elementwise relative error "
          f"(|ref| >= 1e-2 max) {rel:.3g}, ties {ties}")
    assert ties == 0
    assert rq.rq_device_error() == 0


@pytest.mark.parametrize("path", [None, rq.PATH_TABLES])
def test_g2_packed_batch64_fused_argmax(g2, path):
    w = synth.WORKLOADS["packed_b64"]
    packed = rq.rq_pack10(g2["dc"], g2["d"]).cpu().numpy()
    rows = _sample_rows(w.V, 2000, 11)
    assert np.array_equal(packed[rows], oracle.pack10(g2["codes"][rows]))
    err, rel, ties = _batched(g2, w, rq.PACKED10, path)
    print(f"packed_b64 path {path} normwise error {err:.3g}, elementwise relative error "
          f"(|ref| >= 1e-2 max) {rel:.3g}, ties {ties}")
    assert ties == 0


@pytest.mark.parametrize("fmt", [0, 1, 2, 4], ids=["u16", "packed10", "sched", "rot10"])
def test_decode512_bit_exact(g2, fmt):
    w = synth.WORKLOADS["decode512"]
    ids = synth.zipf_ids(w.n_ids, w.V, w.zipf_s, 3)
    codes_dev = {0: lambda: g2["dc"], 1: lambda: rq.rq_pack10(g2["dc"], g2["d"]),
                 2: lambda: rq.rq_prepare_sched(g2["dc"], g2["d"]),
                 4: lambda: rq.rq_prepare_rot10(g2["dc"], g2["d"])}[fmt]()
    out = rq.rq_decode_rows(dev(ids), codes_dev, fmt, g2["dC"], g2["d"], w.decode_scale)
    got = out.view(torch.int16).cpu().numpy().view(np.uint16)
    want = oracle.decode_rows_bf16(ids, g2["codes"], g2["C"], w.decode_scale)
    assert np.array_equal(got, want)


# ------------------------------------------------- RQ MLP matvec (no softcap)

@pytest.mark.parametrize("name", ["mlp_gate_b1", "mlp_down_b1"])
@pytest.mark.parametrize("fmt", [0, 2, 3], ids=["u16", "sched", "u8"])
def test_rq_mlp_matvec(name, fmt):
    """y = W x for an RQ-coded MLP weight W [out x in] (ds = 2, about 10 bits/param with the codebooks):
    the same lookup + sum with V = out features and the softcap off."""
    w = synth.WORKLOADS[name]
    d = rq.dims(w.V, w.D, w.M, w.L, w.K)
    data = synth.make(w)
    C, codes, h = data["C"], data["codes"], data["h"]
    c16 = dev(codes.reshape(w.V, -1))
    dc = {rq.U16: lambda: c16, rq.SCHED: lambda: rq.rq_prepare_sched(c16, d),
          rq.U8: lambda: rq.rq_pack8(c16, d)}[fmt]()
    y, _, _ = rq.rq_logits_from_hidden(dev(h), dev(C), dc, fmt, d, 0.0)
    ref = oracle.logits_direct(codes, C, h)        # the plain definition: W x
    err = assert_logits_close(y.cpu().numpy(), ref)
    print(f"{name} normwise error {err:.3g}")
