"""Host-only checks of the C ABI (no GPU needed, no kernel launched):
the library loads, exports every function ``include/rqlut.h`` declares, its
size arithmetic matches the layouts the header states, and malformed
arguments are rejected before any CUDA call."""
import ctypes
import os
import re

import pytest

import lut_logits_serving_b200 as rq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rqlut.h")


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"RQ_API\s+[\w\s\*]*?\b(rq_\w+)\s*\(", text)))


def test_header_declares_the_abi():
    names = declared_functions()
    for n in ("rq_lut_build", "rq_lut_logits", "rq_decode_rows", "rq_logits_from_hidden",
              "rq_pack10", "rq_device_error", "rq_lut_bytes", "rq_logits_workspace_bytes"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = rq.lib()
    for n in declared_functions():
        assert hasattr(lib, n), n
    # and only the ABI is visible (internal C++ symbols are hidden)
    out = os.popen(f"nm -D --defined-only {rq.LIB_PATH}").read()
    exported = set(re.findall(r" T (\w+)", out))
    assert set(declared_functions()) <= exported
    assert not [s for s in exported if s.startswith("_ZN2rq")]


def test_binding_covers_every_declared_symbol():
    for n in declared_functions():
        assert callable(getattr(rq, n)), n


G2 = rq.dims(256000, 2304, 384, 2, 1024)
TINY = rq.dims(4096, 192, 32, 2, 256)


def test_status_strings():
    assert rq.rq_status_string(0) == "RQ_OK"
    assert rq.rq_status_string(3) == "RQ_ERR_WORKSPACE_TOO_SMALL"
    assert rq.rq_status_string(99) == "RQ_ERR_UNKNOWN"
    assert rq.rq_version() >= 100


def test_code_and_lut_sizes():
    # u16 codes [V][M*L]: 393.216 MB; packed 10-bit rows of 960 bytes
    assert rq.rq_codes_bytes(G2, rq.U16) == 256000 * 768 * 2
    assert rq.rq_codes_bytes(G2, rq.PACKED10) == 256000 * 960
    assert rq.rq_codes_bytes(G2, rq.SCHED) == 256000 * 768 * 2
    assert rq.rq_codes_bytes(TINY, rq.PACKED10) == 4096 * 80
    assert rq.rq_codes_bytes(TINY, rq.U8) == 4096 * 64                        # K = 256: bytes
    assert rq.rq_codes_bytes(G2, rq.U8) == 0                                 # K = 1024: none
    assert rq.rq_codes_bytes(rq.dims(10, 3, 1, 1, 1024), rq.PACKED10) == 10 * 2   # ceil(10/8)
    assert rq.rq_codes_bytes(rq.dims(10, 3, 1, 1, 2048), rq.PACKED10) == 0       # K > 1024
    for B, Bs in ((1, 1), (2, 2), (3, 4), (4, 4), (5, 8), (32, 32), (33, 36), (64, 64)):
        assert rq.rq_lut_token_stride(B) == Bs
        assert rq.rq_lut_bytes(G2, B) == 768 * 1024 * Bs * 4
    assert rq.rq_lut_bytes(G2, 1) == 3145728          # 3.1 MB per token


def test_workspace_sizes():
    # B <= 4 takes the vocabulary-tiled path: partial sums for every chunk
    ws1 = rq.rq_logits_workspace_bytes(G2, 1, rq.U16, False)
    assert ws1 > 0 and ws1 % (256000 * 4) == 0 and ws1 // (256000 * 4) <= 64
    ws1a = rq.rq_logits_workspace_bytes(G2, 1, rq.U16, True)
    assert ws1a > ws1
    # B > 4 reads the table through L2: argmax partials only
    assert rq.rq_logits_workspace_bytes(G2, 32, rq.U16, False) == 0
    assert 0 < rq.rq_logits_workspace_bytes(G2, 32, rq.U16, True) < 1 << 20
    # the fused call adds one token group's table (<= 32 tokens)
    f64 = rq.rq_fused_workspace_bytes(G2, 64, rq.PACKED10, True)
    assert f64 >= rq.rq_lut_bytes(G2, 32)
    assert f64 < rq.rq_lut_bytes(G2, 64)
    # a small shape the tensor-core decode can take: its scratch (split hidden
    # states and codebooks) is larger than an 8-token table, and the fused
    # workspace covers it; a shape it cannot take keeps the table size
    small = rq.dims(1000, 48, 8, 2, 64)
    assert rq.rq_fused_workspace_bytes(small, 8, rq.U16, False) > rq.rq_lut_bytes(small, 8)
    odd = rq.dims(1000, 40, 8, 2, 64)                  # ds = 5
    assert rq.rq_fused_workspace_bytes(odd, 8, rq.U16, False) == rq.rq_lut_bytes(odd, 8)
    # never O(V*M*L) (the pages' naive gather index would be 1.57 GB)
    for B in (1, 2, 3, 4, 5, 32, 64):
        assert rq.rq_logits_workspace_bytes(G2, B, rq.U16, True) < 256000 * 768 * 8


def test_invalid_dims_give_zero_sizes():
    for d in (rq.dims(0, 2304, 384, 2, 1024), rq.dims(10, 2305, 384, 2, 1024),
              rq.dims(10, 2304, 384, 0, 1024), rq.dims(10, 2304, 384, 2, 70000)):
        assert rq.rq_lut_bytes(d, 1) == 0
        assert rq.rq_codes_bytes(d, rq.U16) == 0
    assert rq.rq_lut_bytes(G2, 0) == 0


def _fake(addr):
    return ctypes.c_void_p(addr)


def test_argument_errors_return_before_any_launch():
    lib = rq.lib()
    s = _fake(None)
    null = _fake(None)
    a = _fake(0x10000)          # never dereferenced: every call below returns early
    odd = _fake(0x10004)
    INV, MIS, UNS, WS = 1, 5, 2, 3
    assert lib.rq_lut_build(null, a, G2, 1, a, s) == INV
    assert lib.rq_lut_build(a, a, G2, 0, a, s) == INV
    assert lib.rq_lut_build(a, a, rq.dims(10, 7, 2, 1, 4), 1, a, s) == INV   # D % M != 0
    assert lib.rq_lut_build(a, a, G2, 1, odd, s) == MIS                     # lut 16-B
    assert lib.rq_lut_build(a, a, G2, 4096, a, s) == UNS                    # 4096 x 6 floats > 48 KB
    assert lib.rq_lut_logits(a, 0, G2, a, 1, 30.0, null, null, null, 0, s) == INV
    assert lib.rq_lut_logits(a, 7, G2, a, 1, 30.0, a, null, null, 0, s) == INV
    assert lib.rq_lut_logits(a, 1, rq.dims(10, 8, 4, 2, 2048), a, 1, 30.0, a, null, null, 0,
                             s) == UNS
    assert lib.rq_lut_logits(odd, 0, G2, a, 1, 30.0, a, null, null, 0, s) == MIS
    assert lib.rq_lut_logits(a, 0, G2, odd, 1, 30.0, a, null, null, 0, s) == MIS
    assert lib.rq_logits_from_hidden(a, a, a, 0, G2, 1, 30.0, a, null, null, 0, s) == WS
    assert lib.rq_logits_from_hidden_path(a, a, a, 0, G2, 1, 30.0, a, null, null, 0, 7, s) == INV
    assert lib.rq_argmax_candidates(null, a, 1, 10, 0, a, a, s) == INV
    assert lib.rq_argmax_candidates(a, a, 1, 10, 2**31 - 5, a, a, s) == INV   # int32 rows
    assert lib.rq_argmax_candidates(a, a, 0, 10, 0, a, a, s) == INV
    assert lib.rq_argmax_candidates(_fake(0x10002), a, 1, 10, 0, a, a, s) == MIS
    assert lib.rq_argmax_merge(a, a, 0, 1, a, s) == INV
    assert lib.rq_argmax_merge(a, null, 2, 1, a, s) == INV
    assert lib.rq_argmax_merge(a, a, 2, 1, _fake(0x10002), s) == MIS
    assert lib.rq_logits_from_hidden_path(a, a, a, 0, G2, 1, 30.0, a, null, null, 0, 3, s) == WS
    assert lib.rq_decode_rows(null, 5, a, 0, a, G2, 48.0, a, s) == INV
    assert lib.rq_decode_rows(a, -1, a, 0, a, G2, 48.0, a, s) == INV
    assert lib.rq_decode_rows(null, 0, null, 0, null, G2, 48.0, null, s) == 0   # N = 0: no-op
    assert lib.rq_decode_rows(_fake(0x10002), 5, a, 0, a, G2, 48.0, a, s) == MIS
    assert lib.rq_decode_rows(a, 5, a, 9, a, G2, 48.0, a, s) == INV            # unknown format
    assert lib.rq_decode_rows(a, 5, a, 3, a, G2, 48.0, a, s) == UNS            # u8 codes, K > 256
    assert lib.rq_decode_rows(a, 5, a, 0, _fake(0x10002), G2, 48.0, a, s) == MIS  # C 4-B
    assert lib.rq_decode_rows(a, 5, a, 0, a, G2, 48.0, _fake(0x10001), s) == MIS  # out 2-B
    assert lib.rq_decode_rows(a, 5, _fake(0x10008), 2, a, G2, 48.0, a, s) == MIS  # sched 16-B
    assert lib.rq_pack10(null, G2, a, s) == INV
    assert lib.rq_pack10(_fake(0x10001), G2, a, s) == MIS
    assert lib.rq_device_error(ctypes.POINTER(ctypes.c_uint32)(), 0) == INV   # out NULL
    assert lib.rq_pack8(a, G2, a, s) == UNS                                   # K > 256
    assert lib.rq_prepare_sched(null, G2, a, null, s) == INV
    assert lib.rq_prepare_sched(a, rq.dims(10, 48, 24, 1, 64), _fake(0x900000), null, s) == UNS
    assert lib.rq_prepare_sched(a, G2, _fake(0x10000 + 64), null, s) == INV    # overlap
    assert lib.rq_lut_logits(a, 2, rq.dims(10, 48, 24, 1, 64), a, 1, 30.0, a, null, null, 0,
                             s) == UNS                                        # sched, P % 32
    assert lib.rq_device_error(None, 0) == INV
    assert lib.rq_encode(null, G2, a, a, s) == INV
    big = 1 << 40
    assert lib.rq_topk_sample(a, 256000, 1, 0, 1.0, 0, 0, null, null, a, a, big, s) == INV
    assert lib.rq_topk_sample(a, 256000, 1, 1025, 1.0, 0, 0, null, null, a, a, big, s) == UNS
    assert lib.rq_topk_sample(a, 100, 1, 101, 1.0, 0, 0, null, null, a, a, big, s) == INV
    assert lib.rq_topk_sample(a, 256000, 1, 50, 1.0, 0, 0, null, null, a, a, 16, s) == WS
    assert lib.rq_topk_sample(a, 256000, 1, 50, 1.0, 0, 0, null, null, a, _fake(0x10010), big,
                              s) == MIS
    assert rq.rq_topk_workspace_bytes(256000, 1, 50) > 0
    assert rq.rq_topk_workspace_bytes(256000, 1, 1025) == 0
    assert lib.rq_encode(null, rq.dims(0, 2304, 384, 2, 1024), null, null, s) == 0   # V = 0
    assert lib.rq_encode(a, rq.dims(10, 66, 2, 2, 16), a, _fake(0x900000), s) == UNS   # ds 33
    assert lib.rq_encode(_fake(0x10002), G2, a, _fake(0x90000000), s) == MIS
    assert lib.rq_encode(a, G2, _fake(0x90000000), _fake(0x10000 + 4096), s) == INV   # overlap


def test_python_binding_rejects_cpu_tensors():
    import torch
    h = torch.zeros(1, 192)
    C = torch.zeros(32, 2, 256, 6)
    with pytest.raises(ValueError):
        rq.rq_lut_build(h, C, TINY, lut=torch.zeros(64, 256, 1))


def test_python_binding_checks_buffer_sizes_before_the_call(monkeypatch):
    """A short buffer is refused by name before any pointer reaches the C
    call (the C ABI takes bare pointers and could not tell).  CPU tensors
    stand in for device ones here: the device check is switched off and the
    library's launching calls are replaced by one that only reports being
    reached, so no pointer is ever passed on."""
    import torch
    real = rq.lib()

    class NoLaunch:
        def __getattr__(self, name):
            if name.endswith("_bytes") or name in ("rq_lut_token_stride", "rq_status_string"):
                return getattr(real, name)

            def reached(*a):
                raise RuntimeError(f"{name} reached")
            return reached

    monkeypatch.setattr(rq, "lib", lambda: NoLaunch())
    monkeypatch.setattr(rq, "_on_device", lambda t: True)
    monkeypatch.setattr(rq, "_stream", lambda s: ctypes.c_void_p(None))

    d = TINY                                  # V 4096, D 192, M 32, L 2, K 256
    V, D, P = d.V, d.D, d.M * d.L
    h = torch.zeros(2, D)
    C = torch.zeros(d.M, d.L, d.K, D // d.M)
    codes = torch.zeros((V, P), dtype=torch.uint16)
    lut = torch.zeros(P, d.K, 2)

    def refused(fn, *a, match, **kw):
        with pytest.raises(ValueError, match=match):
            fn(*a, **kw)

    def reaches(fn, *a, **kw):
        with pytest.raises(RuntimeError, match="reached"):
            fn(*a, **kw)

    refused(rq.rq_lut_build, h, C[:-1], d, match="C: .* bytes")
    refused(rq.rq_lut_build, h, C, d, lut=torch.zeros(P, d.K, 1), match="lut: .* bytes")
    refused(rq.rq_lut_build, torch.zeros(2, D + 1), C, d, match=r"h: shape")
    reaches(rq.rq_lut_build, h, C, d, lut=lut)
    refused(rq.rq_lut_logits, codes[:-1], rq.U16, d, lut, 2, match="codes: .* bytes")
    refused(rq.rq_lut_logits, codes, rq.U16, d, lut, 2, logits=torch.zeros(2, V - 1),
            match="logits: .* bytes")
    reaches(rq.rq_lut_logits, codes, rq.U16, d, lut, 2, want_argmax=True)
    refused(rq.rq_logits_from_hidden, h, C, codes, rq.U16, d, logits=torch.zeros(1, V),
            match="logits: .* bytes")
    refused(rq.rq_logits_from_hidden, h, C, codes, rq.U16, d, want_argmax=True,
            logits=torch.zeros(2, V), argmax=torch.zeros(1, dtype=torch.int32),
            match="argmax: .* bytes")
    reaches(rq.rq_logits_from_hidden, h, C, codes, rq.U16, d, want_argmax=True)
    ids = torch.zeros(5, dtype=torch.int32)
    refused(rq.rq_decode_rows, ids, codes, rq.U16, C, d, 1.0,
            out=torch.zeros((4, D), dtype=torch.bfloat16), match="out: .* bytes")
    reaches(rq.rq_decode_rows, ids, codes, rq.U16, C, d, 1.0)
    refused(rq.rq_pack10, codes, d, out=torch.zeros((V, 79), dtype=torch.uint8),
            match="packed: .* bytes")             # a row needs ceil(10 * 64 / 8) = 80 bytes
    reaches(rq.rq_pack10, codes, d)
    refused(rq.rq_greedy_step, h, C, codes, rq.U16, d,
            rows=torch.zeros((1, D), dtype=torch.bfloat16), match="rows: .* bytes")
    reaches(rq.rq_greedy_step, h, C, codes, rq.U16, d)
    refused(rq.rq_topk_sample, torch.zeros(2, 100), 8, token=torch.zeros(1, dtype=torch.int32),
            match="token: .* bytes")
    reaches(rq.rq_topk_sample, torch.zeros(2, 100), 8)
    refused(rq.rq_argmax_merge, torch.zeros(3, 4), torch.zeros((3, 4), dtype=torch.int32),
            out=torch.zeros(3, dtype=torch.int32), match="argmax: .* bytes")
    refused(rq.rq_argmax_candidates, torch.zeros(3, 50), torch.zeros(2, dtype=torch.int32), 0,
            match="argmax: .* bytes")
    refused(rq.rq_encode, torch.zeros(V - 1, D), C, d, match="X: .* bytes")
    reaches(rq.rq_encode, torch.zeros(V, D), C, d)
    refused(rq.rq_prepare_sched, codes, d, out=codes[:-1], match="out: .* bytes")
    reaches(rq.rq_prepare_sched, codes, d)


C_CLIENT = r"""
#include <stdio.h>
#include <string.h>
#include "rqlut.h"

int main(void) {
    rq_dims g2 = {256000, 2304, 384, 2, 1024};
    if (rq_version() <= 0) return 10;
    if (rq_codes_bytes(g2, RQ_CODES_U16) != (size_t)256000 * 768 * 2) return 11;
    if (rq_codes_bytes(g2, RQ_CODES_PACKED10) != (size_t)256000 * 960) return 12;
    if (rq_codes_bytes(g2, RQ_CODES_U8) != 0) return 13;              /* K > 256 */
    if (rq_lut_bytes(g2, 1) != (size_t)768 * 1024 * 4) return 14;
    if (rq_lut_build(NULL, NULL, g2, 1, NULL, NULL) != RQ_ERR_INVALID_ARGUMENT) return 15;
    if (rq_decode_rows(NULL, 0, NULL, RQ_CODES_U16, NULL, g2, 48.0f, NULL, NULL) != RQ_OK)
        return 16;                                                     /* N = 0: no-op */
    if (strlen(rq_status_string(RQ_ERR_MISALIGNED)) == 0) return 17;
    printf("ok\n");
    return 0;
}
"""


def test_header_serves_a_plain_c_client(tmp_path):
    """include/rqlut.h compiles as C99 and C++11 with warnings as errors, and a
    C program linked against the library runs its host-side queries and
    argument checks (no device work, no torch, no Python)."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    inc = os.path.join(ROOT, "include")
    libdir = os.path.dirname(rq.LIB_PATH)
    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", f"-I{inc}", str(src),
                    f"-L{libdir}", "-l:librqlut.so", f"-Wl,-rpath,{libdir}", "-o", str(exe)],
                   check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0 and out.stdout.strip() == "ok", (out.returncode, out.stderr)
    cpp = tmp_path / "client.cpp"
    cpp.write_text('#include "rqlut.h"\nint main() { return rq_version() > 0 ? 0 : 1; }\n')
    subprocess.run(["g++", "-std=c++11", "-Wall", "-Wextra", "-Werror", "-fsyntax-only",
                    f"-I{inc}", str(cpp)], check=True, capture_output=True, text=True)


def test_missing_library_fails_loudly(tmp_path):
    """Without the built library the binding raises; nothing falls back to
    the oracle or to PyTorch."""
    import subprocess
    import sys
    code = ("import lut_logits_serving_b200 as rq\n"
            f"rq.LIB_PATH = {str(tmp_path / 'librqlut.so')!r}\n"
            "try:\n"
            "    rq.rq_version()\n"
            "except RuntimeError as e:\n"
            "    print('raised:', 'no CPU fallback' in str(e))\n"
            "else:\n"
            "    print('returned')\n")
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                         cwd=ROOT, timeout=120)
    assert out.stdout.strip() == "raised: True", (out.stdout, out.stderr[-500:])


def test_product_code_does_not_reach_the_oracle():
    """Only tests, smoke() and the bench's CPU legs may load the oracle: the
    package's sources never import it."""
    pkg = os.path.join(ROOT, "lut_logits_serving_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", text, re.M), f
                assert "rq_oracle" not in text and "librq_oracle" not in text, f
