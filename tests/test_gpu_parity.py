"""GPU parity: the CUDA path, called through the C ABI, against the CPU
oracle on the same seeded inputs, element by element.  Small shapes that
span several tiles and chunks with ragged tails, every kernel path (the
shared-memory vocabulary-tiled pass for B <= 4, the L2-served token-group
pass, the generic fallback), both code formats, and the degenerate cases."""
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


def make_case(V, D, M, L, K, B, seed=0, sigmas=(0.05, 0.01), hscale=1.0):
    C = synth.codebooks(M, L, K, D // M, sigmas, seed)
    codes = synth.codes(V, M, L, K, seed + 1)
    h = synth.hidden(B, D, hscale, seed + 2)
    return C, codes, h


def oracle_logits(C, codes, h, cap):
    T = oracle.lut_build(h, C, "f64")
    return oracle.softcap(oracle.logits_lut(codes, T), cap)


def gpu_codes(codes, fmt, d):
    c16 = dev(codes.reshape(codes.shape[0], -1))
    if fmt == rq.U16:
        return c16
    if fmt == rq.SCHED:
        return rq.rq_prepare_sched(c16, d)
    if fmt == rq.U8:
        return rq.rq_pack8(c16, d)
    if fmt == rq.ROT10:
        return rq.rq_prepare_rot10(c16, d)
    return rq.rq_pack10(c16, d)


def fmt_applies(fmt, M, L, K):
    if fmt == rq.PACKED10:
        return K <= 1024
    if fmt == rq.SCHED:
        return K <= 1024 and (M * L) % 32 == 0
    if fmt == rq.U8:
        return K <= 256
    if fmt == rq.ROT10:
        return K <= 1024 and (M * L) % 64 == 0
    return True


# ------------------------------------------------------------- lut build

@pytest.mark.parametrize("B", [1, 2, 3, 4, 5, 8, 32])
def test_lut_build_matches_oracle(B):
    V, D, M, L, K = 64, 192, 32, 2, 256
    C, _, h = make_case(V, D, M, L, K, B)
    d = rq.dims(V, D, M, L, K)
    lut = rq.rq_lut_build(dev(h), dev(C), d).cpu().numpy()
    Bs = rq.rq_lut_token_stride(B)
    assert lut.shape == (M * L, K, Bs)
    T = oracle.lut_build(h, C, "f64")                      # [B, M, L, K]
    ref = T.reshape(B, M * L, K).transpose(1, 2, 0)        # [P, K, B]
    scale = np.max(np.abs(ref))
    assert np.max(np.abs(lut[:, :, :B] - ref)) <= 2e-6 * scale
    assert np.all(lut[:, :, B:] == 0)                      # padding tokens are zero
    torch.cuda.synchronize()


# ------------------------------------------------------------ the logits

CASES = [
    # V,    D,   M,  L, K,    note
    (4096, 192, 32, 2, 256),   # the tiny workload
    (4099, 192, 32, 2, 256),   # ragged last tile
    (257, 48, 8, 2, 64),       # one row past a tile
    (1, 48, 8, 2, 64),         # a single row
    (3000, 288, 48, 2, 1024),  # K = 1024 instances, P = 96 -> 3 chunks (40, 40, 16)
    (2000, 96, 16, 3, 100),    # L = 3, non-power-of-two K (clamped codes path)
    (1500, 64, 64, 1, 32),     # ds = 1, L = 1
    (700, 9, 3, 1, 7),         # P = 3: generic fallback
    (1200, 128, 64, 1, 100),   # scheduled table stride 128 (two CTAs per SM)
    (900, 96, 16, 2, 300),     # scheduled table stride 512
    (600, 64, 32, 2, 37),      # scheduled table stride 64
    (2600, 384, 64, 2, 1024),  # K = 1024, P = 128: 10-bit slices at both window offsets
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "V%d_D%d_M%d_L%d_K%d" % c)
@pytest.mark.parametrize("B", [1, 2, 3, 4, 5, 13, 32, 33])
@pytest.mark.parametrize("fmt", [0, 1, 2, 3, 4], ids=["u16", "packed10", "sched", "u8", "rot10"])
def test_logits_and_argmax(case, B, fmt):
    V, D, M, L, K = case
    if not fmt_applies(fmt, M, L, K):
        pytest.skip("format does not hold this shape")
    C, codes, h = make_case(V, D, M, L, K, B, seed=V + B)
    d = rq.dims(V, D, M, L, K)
    cap = 30.0
    ref = oracle_logits(C, codes, h, cap)
    dc = gpu_codes(codes, fmt, d)
    dh, dC = dev(h), dev(C)
    lut = rq.rq_lut_build(dh, dC, d)
    logits, am, _ = rq.rq_lut_logits(dc, fmt, d, lut, B, cap, want_argmax=True)
    got = logits.cpu().numpy()
    assert got.shape == (B, V)
    assert_logits_close(got, ref)
    check_argmax(am.cpu().numpy(), ref)
    # the fused call gives the same numbers
    logits2, am2, _ = rq.rq_logits_from_hidden(dh, dC, dc, fmt, d, cap, want_argmax=True)
    assert_logits_close(logits2.cpu().numpy(), ref)
    check_argmax(am2.cpu().numpy(), ref)      # (B >= 8 may sum in the decode order)
    # argmax alone (logits not written) agrees
    _, am3, _ = rq.rq_lut_logits(dc, fmt, d, lut, B, cap, want_logits=False, want_argmax=True)
    assert np.array_equal(am3.cpu().numpy(), am.cpu().numpy())
    assert rq.rq_device_error() == 0


def test_u16_and_packed_agree_bit_for_bit_on_the_generic_order():
    """Both formats feed the same lookups in the same order in the L2-served
    pass, so their logits are identical."""
    V, D, M, L, K, B = 2048, 192, 32, 2, 256, 8
    C, codes, h = make_case(V, D, M, L, K, B)
    d = rq.dims(V, D, M, L, K)
    lut = rq.rq_lut_build(dev(h), dev(C), d)
    a, _, _ = rq.rq_lut_logits(gpu_codes(codes, 0, d), 0, d, lut, B, 30.0)
    b, _, _ = rq.rq_lut_logits(gpu_codes(codes, 1, d), 1, d, lut, B, 30.0)
    assert torch.equal(a, b)


def test_softcap_off_gives_raw_sums():
    V, D, M, L, K, B = 1024, 192, 32, 2, 256, 1
    C, codes, h = make_case(V, D, M, L, K, B, hscale=20.0)   # large logits
    d = rq.dims(V, D, M, L, K)
    T = oracle.lut_build(h, C, "f64")
    z = oracle.logits_lut(codes, T)
    assert np.max(np.abs(z)) > 30.0        # the softcap would have bent these
    lut = rq.rq_lut_build(dev(h), dev(C), d)
    got, _, _ = rq.rq_lut_logits(dev(codes.reshape(V, -1)), 0, d, lut, B, 0.0)
    assert_logits_close(got.cpu().numpy(), z)
    capped, _, _ = rq.rq_lut_logits(dev(codes.reshape(V, -1)), 0, d, lut, B, 30.0)
    assert float(capped.abs().max()) < 30.0


def test_single_codeword_ties_go_to_index_zero():
    """K = 1: every row is the same vector, all logits are bit-identical and
    the argmax is row 0 on every path."""
    V, D, M, L, K = 3000, 96, 16, 2, 1
    for B in (1, 3, 8):
        C, codes, h = make_case(V, D, M, L, K, B)
        d = rq.dims(V, D, M, L, K)
        lut = rq.rq_lut_build(dev(h), dev(C), d)
        for fmt in (0, 1, 2):
            logits, am, _ = rq.rq_lut_logits(gpu_codes(codes, fmt, d), fmt, d, lut, B, 30.0,
                                             want_argmax=True)
            lg = logits.cpu().numpy()
            assert np.all(lg == lg[:, :1])
            assert np.all(am.cpu().numpy() == 0)


def test_planted_maximum_is_found_at_every_position():
    """One row holds a unique maximum; the argmax must find it wherever it
    sits (first row, last row, tile and chunk boundaries)."""
    V, D, M, L, K, B = 5000, 96, 16, 2, 16, 1
    rng = np.random.default_rng(1)
    C = synth.codebooks(M, L, K, D // M, (0.05, 0.01), 0)
    h = synth.hidden(1, D, 1.0, 2)
    T = oracle.lut_build(h, C, "f64")[0]                   # [M, L, K]
    best = np.argmax(T, axis=2)                            # best code per table
    worst = np.argmin(T, axis=2)
    d = rq.dims(V, D, M, L, K)
    lut = rq.rq_lut_build(dev(h), dev(C), d)
    for pos in (0, 1, 255, 256, 2047, 4095, 4999):
        codes = np.broadcast_to(worst, (V, M, L)).copy().astype(np.uint16)
        codes[rng.integers(0, V, 50)] = rng.integers(0, K, (50, M, L))
        codes[pos] = best
        for fmt in (0, 1, 2):
            _, am, _ = rq.rq_lut_logits(gpu_codes(codes, fmt, d), fmt, d, lut, B, 30.0,
                                        want_logits=False, want_argmax=True)
            assert int(am.cpu()[0]) == pos


def test_out_of_range_codes_stay_in_bounds():
    """Codes >= K never index outside the tables: modulo K for a power of
    two, clamped to K-1 otherwise (the header's stated behaviour)."""
    V, D, M, L = 600, 48, 8, 2
    for K, fix in ((64, lambda c: c % 64), (100, lambda c: np.minimum(c, 99))):
        C, _, h = make_case(V, D, M, L, K, 1)
        rng = np.random.default_rng(3)
        raw = rng.integers(0, 65536, (V, M, L)).astype(np.uint16)
        d = rq.dims(V, D, M, L, K)
        lut = rq.rq_lut_build(dev(h), dev(C), d)
        got, _, _ = rq.rq_lut_logits(dev(raw.reshape(V, -1)), 0, d, lut, 1, 30.0)
        ref = oracle_logits(C, fix(raw.astype(np.int64)).astype(np.uint16), h, 30.0)
        assert_logits_close(got.cpu().numpy(), ref)


def unrotate10(buf, V, P):
    """The RQ_CODES_PACKED10_ROT bytes back to uint16 codes [V, P], from the
    layout's definition: V packed rows of 10 P / 8 bytes (code slot q at bits
    [10q, 10q + 10), LSB first), then the rotations uint8 [P / 32][V]; slot j of
    slice s holds pair 32 s + (j + r) mod 32."""
    rb = P // 8 * 10
    rows = np.asarray(buf[:V * rb], np.uint8).reshape(V, rb)
    rot = np.asarray(buf[V * rb:V * rb + V * (P // 32)], np.uint8).reshape(P // 32, V) & 31
    bits = np.unpackbits(rows, axis=1, bitorder="little").reshape(V, P, 10).astype(np.int64)
    slots = (bits << np.arange(10)).sum(axis=2)                       # [V, P] by slot
    out = np.empty((V, P), np.int64)
    j = np.arange(32)
    for sl in range(P // 32):
        pair = 32 * sl + (j[None, :] + rot[sl][:, None].astype(np.int64)) % 32
        np.put_along_axis(out, pair, slots[:, 32 * sl:32 * sl + 32], axis=1)
    return out


@pytest.mark.parametrize("V,P,K", [(4099, 64, 256), (1000, 128, 1024), (33, 192, 100)])
def test_rotated_layout_holds_the_codes(V, P, K):
    """rq_prepare_rot10 writes every row's codes, each slice rotated by its own
    byte, and its rotations leave fewer bank passes than the plain order."""
    codes = synth.codes(V, P // 2, 2, K, V)
    d = rq.dims(V, 6 * (P // 2), P // 2, 2, K)
    buf, (steps, passes) = rq.rq_prepare_rot10(dev(codes.reshape(V, -1)), d, stats=True)
    assert buf.numel() == rq.rq_codes_bytes(d, rq.ROT10) == V * (P // 8 * 10 + P // 32)
    got = unrotate10(buf.cpu().numpy(), V, P)
    assert np.array_equal(got, codes.reshape(V, -1).astype(np.int64))
    assert steps == 32 * ((V + 31) // 32) * (P // 32)
    if K % 32 == 0 and V >= 1000:
        # plain order: ~3.5 passes per step for random codes
        assert passes / steps < 3.0


# ------------------------------------------------------------ row decode

@pytest.mark.parametrize("fmt", [0, 1, 2, 3, 4], ids=["u16", "packed10", "sched", "u8", "rot10"])
@pytest.mark.parametrize("shape", [(4096, 192, 32, 2, 256), (5000, 288, 48, 2, 1024),
                                   (300, 96, 16, 3, 100), (50, 9, 3, 1, 7)])
def test_decode_rows_bit_exact(shape, fmt):
    V, D, M, L, K = shape
    if not fmt_applies(fmt, M, L, K):
        pytest.skip("format does not hold this shape")
    C, codes, _ = make_case(V, D, M, L, K, 1, sigmas=(0.02, 0.005))
    ids = synth.zipf_ids(257, V, 1.1, 3)
    d = rq.dims(V, D, M, L, K)
    scale = float(np.sqrt(D))
    out = rq.rq_decode_rows(dev(ids), gpu_codes(codes, fmt, d), fmt, dev(C), d, scale)
    got = out.view(torch.int16).cpu().numpy().view(np.uint16)
    want = oracle.decode_rows_bf16(ids, codes, C, scale)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("shift_out,shift_C", [(0, 0), (1, 0), (0, 1)],
                         ids=["aligned", "odd_out", "odd_C"])
def test_decode_rows_ragged_subspace_blocks_and_odd_pointers(shift_out, shift_C):
    """M = 200 spans two blocks of the pair kernel with a ragged second one;
    an output 2 bytes off a 4-byte boundary, or codebooks 4 bytes off an
    8-byte one, take the one-thread-per-subspace kernel, bit for bit alike."""
    V, D, M, L, K = 3000, 1200, 200, 2, 512
    C, codes, _ = make_case(V, D, M, L, K, 1, sigmas=(0.02, 0.005))
    ids = synth.zipf_ids(129, V, 1.1, 5)
    d = rq.dims(V, D, M, L, K)
    cbuf = torch.empty(C.size + 1, dtype=torch.float32, device="cuda")
    dC = cbuf[shift_C:shift_C + C.size].view(C.shape)
    dC.copy_(dev(C))
    obuf = torch.full((len(ids) * D + 1,), float("nan"), dtype=torch.bfloat16, device="cuda")
    out = obuf[shift_out:shift_out + len(ids) * D].view(len(ids), D)
    rq.rq_decode_rows(dev(ids), dev(codes.reshape(V, -1)), rq.U16, dC, d, 7.0, out=out)
    got = out.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, oracle.decode_rows_bf16(ids, codes, C, 7.0))
    assert rq.rq_device_error() == 0


@pytest.mark.parametrize("N", [389, 1003])
def test_decode_rows_several_rows_per_thread(N):
    """At D = 2304, M = 384, 389 ids take two rows per thread and 1003 ids four
    (the grid of one row per thread would not be resident in one wave), with a
    ragged last block and bad ids inside a thread's group of rows."""
    V, D, M, L, K = 700, 2304, 384, 2, 1024
    C, codes, _ = make_case(V, D, M, L, K, 1, sigmas=(0.02, 0.005))
    ids = synth.zipf_ids(N, V, 1.1, 11)
    bad = [5, N // 2, N - 1]
    ids[bad] = [-3, V, V + 1000]
    d = rq.dims(V, D, M, L, K)
    rq.rq_device_error(clear=True)
    out = torch.full((N, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    rq.rq_decode_rows(dev(ids), dev(codes.reshape(V, -1)), rq.U16, dev(C), d, 48.0, out=out)
    got = out.view(torch.int16).cpu().numpy().view(np.uint16)
    good = np.setdiff1d(np.arange(N), bad)
    assert np.all(got[bad] == 0)
    assert np.array_equal(got[good], oracle.decode_rows_bf16(ids[good], codes, C, 48.0))
    assert rq.rq_device_error(clear=True) == 2


def test_decode_rows_bad_ids_give_zero_rows_and_a_device_error():
    V, D, M, L, K = 100, 48, 8, 2, 16
    C, codes, _ = make_case(V, D, M, L, K, 1)
    d = rq.dims(V, D, M, L, K)
    rq.rq_device_error(clear=True)
    ids = np.array([3, -1, 100, 99], np.int32)
    out = rq.rq_decode_rows(dev(ids), dev(codes.reshape(V, -1)), 0, dev(C), d, 1.0)
    got = out.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.all(got[1] == 0) and np.all(got[2] == 0)
    want = oracle.decode_rows_bf16(np.array([3, 99], np.int32), codes, C, 1.0)
    assert np.array_equal(got[[0, 3]], want)
    assert rq.rq_device_error(clear=True) == 2
    assert rq.rq_device_error() == 0


def test_decode_rows_empty_is_a_noop():
    d = rq.dims(10, 8, 4, 2, 4)
    lib = rq.lib()
    assert lib.rq_decode_rows(None, 0, None, 0, None, d, 1.0, None, None) == 0


# ---------------------------------------------------------------- packing

@pytest.mark.parametrize("P", [(32, 2), (3, 1), (7, 3), (384, 2)])
def test_pack10_matches_oracle(P):
    M, L = P
    V = 777
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 1024, (V, M, L)).astype(np.uint16)
    d = rq.dims(V, 8 * M, M, L, 1024)
    got = rq.rq_pack10(dev(codes.reshape(V, -1)), d).cpu().numpy()
    assert np.array_equal(got, oracle.pack10(codes))


# ------------------------------------------------------ scheduled codes

def _sched_shift(K):
    """The entry shift the header defines: table stride 2^s, the smallest
    power of two >= K and at least 32."""
    s = 5
    while (1 << s) < K:
        s += 1
    return s


@pytest.mark.parametrize("shape", [(4096, 192, 32, 2, 256), (1000, 96, 16, 2, 1024),
                                   (77, 96, 32, 1, 64), (3000, 288, 48, 2, 1024),
                                   (500, 64, 32, 2, 16), (700, 64, 32, 1, 37),
                                   (900, 128, 64, 1, 100), (333, 64, 32, 2, 300)])
def test_prepare_sched_is_a_permutation_within_groups(shape):
    """Chunk-major [P/32][V][32]; every row's 32-entry slice holds exactly
    the slice's 32 (position, code) pairs, each once, as i << s | c."""
    V, D, M, L, K = shape
    sh = _sched_shift(K)
    codes = synth.codes(V, M, L, K, 4)
    d = rq.dims(V, D, M, L, K)
    P = M * L
    out, (steps, passes) = rq.rq_prepare_sched(dev(codes.reshape(V, -1)), d, stats=True)
    raw = out.view(torch.int16).cpu().numpy().view(np.uint16).astype(np.int64)
    assert raw.size == V * P
    e = raw.reshape(P // 32, V, 32).transpose(1, 0, 2)     # [V, P/32, 32]
    assert np.all(e >> (sh + 5) == 0)
    pos = e >> sh
    code = e & ((1 << sh) - 1)
    order = np.argsort(pos, axis=2, kind="stable")
    assert np.array_equal(np.take_along_axis(pos, order, 2),
                          np.broadcast_to(np.arange(32), pos.shape))
    assert np.array_equal(np.take_along_axis(code, order, 2), codes.reshape(V, P // 32, 32))
    assert steps == 32 * ((V + 31) // 32) * (P // 32)
    assert passes >= steps


def test_prepare_sched_quality_on_random_codes():
    """Random codes cost ~3.5 shared-memory passes per lookup step in their
    natural order; the schedule must bring the average below 1.6."""
    V, D, M, L, K = 20000, 2304, 384, 2, 1024
    codes = synth.codes(V, M, L, K, 1)
    d = rq.dims(V, D, M, L, K)
    _, (steps, passes) = rq.rq_prepare_sched(dev(codes.reshape(V, -1)), d, stats=True)
    flat = codes.reshape(V, -1)
    # a warp's step k: 32 rows, code k of each row's slice of chunk c
    natural = np.mean([np.bincount(flat[r:r + 32, 32 * c + k] & 31, minlength=32).max()
                       for r in range(0, 2000, 32) for c in range(4) for k in range(32)])
    print(f"bank passes per step: natural order {natural:.2f}, scheduled {passes / steps:.2f}")
    assert passes / steps < 1.6
    assert natural > 2.5


def test_prepare_sched_rejects_unsupported_shapes():
    d = rq.dims(100, 48, 24, 1, 1024)          # M*L = 24: not a multiple of 32
    c = torch.zeros((100, 24), dtype=torch.uint16, device="cuda")
    with pytest.raises(rq.RqError):
        rq.rq_prepare_sched(c, d)
    d2 = rq.dims(100, 64, 32, 1, 2048)         # K > 1024
    c2 = torch.zeros((100, 32), dtype=torch.uint16, device="cuda")
    with pytest.raises(rq.RqError):
        rq.rq_prepare_sched(c2, d2)
    with pytest.raises(rq.RqError):            # in place is refused
        rq.rq_prepare_sched(c2, rq.dims(100, 64, 32, 1, 1024), out=c2)


# ------------------------------------------------------------ greedy step

@pytest.mark.parametrize("B", [1, 3, 5, 33])
@pytest.mark.parametrize("fmt", [0, 1, 2, 3, 4], ids=["u16", "packed10", "sched", "u8", "rot10"])
def test_greedy_step_rows_are_the_picked_tokens_rows(B, fmt):
    V, D, M, L, K = 3000, 192, 32, 2, 256
    C, codes, h = make_case(V, D, M, L, K, B, seed=B)
    d = rq.dims(V, D, M, L, K)
    dc = gpu_codes(codes, fmt, d)
    ref = oracle_logits(C, codes, h, 30.0)
    logits, am, rows, _ = rq.rq_greedy_step(dev(h), dev(C), dc, fmt, d, 30.0, scale=8.0)
    assert_logits_close(logits.cpu().numpy(), ref)
    check_argmax(am.cpu().numpy(), ref)
    ids = am.cpu().numpy().astype(np.int32)
    want = oracle.decode_rows_bf16(ids, codes, C, 8.0)
    assert np.array_equal(rows.view(torch.int16).cpu().numpy().view(np.uint16), want)
    # without logits: same picks and rows
    _, am2, rows2, _ = rq.rq_greedy_step(dev(h), dev(C), dc, fmt, d, 30.0, scale=8.0,
                                         want_logits=False)
    assert torch.equal(am2, am) and torch.equal(rows2, rows)
    assert rq.rq_device_error() == 0


# --------------------------------------- batched rows decoded in shared memory

@pytest.mark.parametrize("V,M,K,B", [
    (1, 8, 64, 8),            # a single row
    (255, 8, 1024, 9),        # fewer rows than one CTA's share
    (148 * 1024 + 7, 16, 300, 32),   # every CTA two tiles, K not a power of two
    (5000, 40, 7, 33),        # 5 code groups, a one-token second group (table path)
    (3001, 16, 1024, 64),     # two full token groups
    (2500, 8, 256, 48),       # a full group (decoded) and a 16-token group (tables)
    (7001, 16, 1024, 64),     # one 64-token group on the tensor cores
    (3333, 8, 512, 100),      # groups of 64 and 32 and a 4-token rest
    (999, 24, 13, 64),        # K < 16: a 64-token group (the workspace holds its scratch)
    (4099, 16, 256, 20),      # one partial group: the tensor cores by default (>= 17 tokens)
    (3000, 8, 1024, 57),      # 32 + a 25-token partial group on the tensor cores
    (4100, 40, 64, 32),       # M = 40: accumulation chains of 16, 16 and 8 subspaces
])
@pytest.mark.parametrize("path", [None, rq.PATH_TABLES, rq.PATH_DECODE_FP32, rq.PATH_DECODE_TC])
def test_fused_decode_paths(V, M, K, B, path):
    """Full 32-token groups with uint16 codes, ds = 6, L = 2, M % 8 == 0: the
    fused call decodes rows (FP32 FMAs or tcgen05 MMAs) or reads tables, as
    asked; groups of fewer tokens use the tables.  Logits and argmax meet the
    same bounds on every path, with both kinds of group in one call."""
    D, L = 6 * M, 2
    C, codes, h = make_case(V, D, M, L, K, B, seed=V + B)
    d = rq.dims(V, D, M, L, K)
    ref = oracle_logits(C, codes, h, 30.0)
    args = (dev(h), dev(C), dev(codes.reshape(V, -1)), rq.U16, d, 30.0)
    # (the fused workspace covers the tensor-core scratch for every shape the
    # kernel takes, so small K and small groups are served as well)
    out = torch.full((B, V), float("nan"), device="cuda")   # stale memory cannot pass
    logits, am, _ = rq.rq_logits_from_hidden(*args, want_argmax=True, logits=out, path=path)
    assert rq.rq_device_error() == 0
    assert_logits_close(logits.cpu().numpy(), ref)
    check_argmax(am.cpu().numpy(), ref)


@pytest.mark.parametrize("V,M,K,B", [
    (4096, 32, 256, 32),      # the tiny workload's shape, one 32-token group
    (5003, 32, 1024, 64),     # one 64-token group, ragged rows
    (2222, 64, 100, 70),      # groups of 64 + a 6-token rest (tables), K not a power of two
    (160000, 32, 256, 40),    # full 1024-row passes of a 32-token group, then an 8-token group
])
def test_packed_codes_on_the_tensor_cores(V, M, K, B):
    """10-bit packed codes (M % 32 == 0) are unpacked by the tensor-core kernel's
    decoders: logits and argmax as for uint16 codes, codes >= K clamped."""
    D = 6 * M
    C, codes, h = make_case(V, D, M, 2, K, B, seed=V + 7)
    d = rq.dims(V, D, M, 2, K)
    ref = oracle_logits(C, codes, h, 30.0)
    packed = rq.rq_pack10(dev(codes.reshape(V, -1)), d)
    out = torch.full((B, V), float("nan"), device="cuda")
    logits, am, _ = rq.rq_logits_from_hidden(dev(h), dev(C), packed, rq.PACKED10, d, 30.0,
                                             want_argmax=True, logits=out,
                                             path=rq.PATH_DECODE_TC)
    assert rq.rq_device_error() == 0
    assert_logits_close(logits.cpu().numpy(), ref)
    check_argmax(am.cpu().numpy(), ref)
    # the default takes the same kernel for the full groups (a rest of fewer
    # than 17 tokens reads its tables) and gives the same numbers there
    logits2, _, _ = rq.rq_logits_from_hidden(dev(h), dev(C), packed, rq.PACKED10, d, 30.0)
    full = B - B % 32 if B % 32 < 17 else B
    assert torch.equal(logits2[:full], logits[:full])
    assert_logits_close(logits2.cpu().numpy(), ref)


@pytest.mark.parametrize("V,M,K,B", [
    (4096, 32, 256, 32),      # two 16-subspace slices, one 32-token group
    (5003, 16, 1024, 64),     # one slice, one 64-token group, ragged rows
    (2222, 48, 100, 70),      # three slices, K not a power of two (7-bit table stride)
    (160000, 32, 256, 40),    # full 1024-row passes of a 32-token group, then 8 tokens
])
def test_scheduled_codes_on_the_tensor_cores(V, M, K, B):
    """Bank-scheduled codes (M % 16 == 0) are put back in pair order by the
    tensor-core kernel's decoders as each stage lands: the logits are those of
    the same codes as drawn, bit for bit, and match the oracle."""
    D = 6 * M
    C, codes, h = make_case(V, D, M, 2, K, B, seed=V + 11)
    d = rq.dims(V, D, M, 2, K)
    ref = oracle_logits(C, codes, h, 30.0)
    c16 = dev(codes.reshape(V, -1))
    sched = rq.rq_prepare_sched(c16, d)
    out = torch.full((B, V), float("nan"), device="cuda")
    logits, am, _ = rq.rq_logits_from_hidden(dev(h), dev(C), sched, rq.SCHED, d, 30.0,
                                             want_argmax=True, logits=out,
                                             path=rq.PATH_DECODE_TC)
    assert rq.rq_device_error() == 0
    assert_logits_close(logits.cpu().numpy(), ref)
    check_argmax(am.cpu().numpy(), ref)
    plain, am_u, _ = rq.rq_logits_from_hidden(dev(h), dev(C), c16, rq.U16, d, 30.0,
                                              want_argmax=True, path=rq.PATH_DECODE_TC)
    assert torch.equal(logits, plain)
    assert torch.equal(am, am_u)
    # the default takes the tensor cores for the full groups of this layout too
    logits2, _, _ = rq.rq_logits_from_hidden(dev(h), dev(C), sched, rq.SCHED, d, 30.0)
    full = B - B % 32 if B % 32 < 17 else B
    assert torch.equal(logits2[:full], logits[:full])


@pytest.mark.parametrize("B", [32, 64])
def test_tensor_core_decode_argmax_only_and_softcap_off(B):
    """Without a logits buffer the tensor-core kernel still leaves the argmax
    partials; with the softcap off it returns the raw sums."""
    V, M, K = 3001, 16, 256
    C, codes, h = make_case(V, 6 * M, M, 2, K, B, seed=11, hscale=20.0)   # logits well past 30
    d = rq.dims(V, 6 * M, M, 2, K)
    args = (dev(h), dev(C), dev(codes.reshape(V, -1)), rq.U16, d)
    ref = oracle_logits(C, codes, h, 30.0)
    _, am, _ = rq.rq_logits_from_hidden(*args, 30.0, want_logits=False, want_argmax=True,
                                        path=rq.PATH_DECODE_TC)
    check_argmax(am.cpu().numpy(), ref)
    raw = oracle_logits(C, codes, h, 0.0)
    assert np.abs(raw).max() > 30.0
    logits, am0, _ = rq.rq_logits_from_hidden(*args, 0.0, want_argmax=True, path=rq.PATH_DECODE_TC)
    assert_logits_close(logits.cpu().numpy(), raw)
    check_argmax(am0.cpu().numpy(), raw)
    assert rq.rq_device_error() == 0


def test_decode_paths_need_their_format():
    """A decode path the format cannot take is refused, not silently replaced."""
    V, M, K, B = 512, 8, 256, 32
    C, codes, h = make_case(V, 6 * M, M, 2, K, B)
    d = rq.dims(V, 6 * M, M, 2, K)
    packed = rq.rq_pack10(dev(codes.reshape(V, -1)), d)
    for path in (rq.PATH_DECODE_FP32, rq.PATH_DECODE_TC):
        with pytest.raises(rq.RqError, match="UNSUPPORTED"):
            rq.rq_logits_from_hidden(dev(h), dev(C), packed, rq.PACKED10, d, 30.0, path=path)
    # the default and the tables serve it
    ref = oracle_logits(C, codes, h, 30.0)
    for path in (None, rq.PATH_TABLES):
        logits, _, _ = rq.rq_logits_from_hidden(dev(h), dev(C), packed, rq.PACKED10, d, 30.0,
                                                path=path)
        assert_logits_close(logits.cpu().numpy(), ref)


@pytest.mark.parametrize("path", [rq.PATH_DECODE_FP32, rq.PATH_DECODE_TC])
def test_fused_decode_clamps_out_of_range_codes(path):
    """Codes >= K read codeword K-1 (non-power-of-two K), as in the other paths."""
    V, M, K, B = 2000, 8, 100, 32
    C, codes, h = make_case(V, 6 * M, M, 2, K, B, seed=3)
    bad = codes.copy()
    bad[::7, :, 1] = 1000
    d = rq.dims(V, 6 * M, M, 2, K)
    ref = oracle_logits(C, np.minimum(bad, K - 1), h, 30.0)
    logits, _, _ = rq.rq_logits_from_hidden(dev(h), dev(C), dev(bad.reshape(V, -1)), rq.U16, d,
                                            30.0, path=path)
    assert_logits_close(logits.cpu().numpy(), ref)


@pytest.mark.parametrize("B", [9, 12, 20, 24, 28, 31])
def test_l2_pass_with_an_exactly_sized_table(B):
    """Token counts whose lane groups are not a power of two: the table is
    allocated to exactly [P][K][Bs] (no workspace after it), so every read
    must stay inside it."""
    V, D, M, L, K = 3000, 192, 32, 2, 256
    C, codes, h = make_case(V, D, M, L, K, B, seed=B)
    d = rq.dims(V, D, M, L, K)
    Bs = rq.rq_lut_token_stride(B)
    lut = torch.empty((M * L, K, Bs), dtype=torch.float32, device="cuda")
    rq.rq_lut_build(dev(h), dev(C), d, lut=lut)
    logits, am, _ = rq.rq_lut_logits(dev(codes.reshape(V, -1)), rq.U16, d, lut, B, 30.0,
                                     want_argmax=True)
    ref = oracle_logits(C, codes, h, 30.0)
    assert_logits_close(logits.cpu().numpy(), ref)
    check_argmax(am.cpu().numpy(), ref)


def test_pack8_round_trip_and_decode():
    """RQ_CODES_U8 holds each code in one byte; rows rebuilt from it are the
    oracle's, bit for bit."""
    V, D, M, L, K = 3000, 96, 16, 2, 200
    C, codes, _ = make_case(V, D, M, L, K, 1, seed=9)
    d = rq.dims(V, D, M, L, K)
    u8 = rq.rq_pack8(dev(codes.reshape(V, -1)), d)
    assert np.array_equal(u8.cpu().numpy(), codes.reshape(V, -1).astype(np.uint8))
    ids = synth.zipf_ids(300, V, 1.1, 4)
    out = rq.rq_decode_rows(dev(ids), u8, rq.U8, dev(C), d, 5.0)
    want = oracle.decode_rows_bf16(ids, codes, C, 5.0)
    assert np.array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), want)
    with pytest.raises(rq.RqError):             # K > 256 has no byte form
        rq.rq_pack8(dev(codes.reshape(V, -1)), rq.dims(V, D, M, L, 300))
