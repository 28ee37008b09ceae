"""Planted mistakes: each mutation below is a plausible slip in the oracle
(transposed operand, dropped term, wrong sign, wrong index split, wrong
rounding, wrong bit order, wrong tie-break, wrong softcap, encoder
residual / codebook / sign slips).  A mutated copy
of the oracle source is compiled on the CPU and the pin checks must catch
every one of them.  The oracle itself is never modified."""
import os
import shutil
import subprocess
import tempfile
import ctypes

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "rq_oracle.c")

MUTATIONS = {
    "transposed_code_index": ("cr[m * L + l]", "cr[l * M + m]"),
    "dropped_level": ("for (int l = 0; l < L; ++l)", "for (int l = 0; l < 1; ++l)"),
    "wrong_sign_lookup": ("acc += T[", "acc -= T["),
    "wrong_subspace_split": ("int m = i / ds, j = i % ds;", "int m = i % M, j = i / M;"),
    "lut_hidden_offset": ("(size_t)m * ds;", "(size_t)m;"),
    "bf16_truncates": ("upper += 1u;", "upper += 0u;"),
    "pack_msb_first": ("(1u << (bit % 8))", "(1u << (7 - bit % 8))"),
    "argmax_last_tie": ("if (y[i] > y[best])", "if (y[i] >= y[best])"),
    "softcap_inverted": ("cap * tanh(y[i] / cap)", "cap * tanh(y[i] * cap)"),
    "decode_scale_before_sum": ("float s = e * scale;", "float s = e * scale * scale;"),
    "encode_no_residual": ("r[j] = r[j] - book[(size_t)best * ds + j];",
                           "r[j] = r[j] - 0.0f * book[(size_t)best * ds + j];"),
    "encode_last_tie": ("if (acc < bestd) {", "if (acc <= bestd) {"),
    "encode_level0_book": ("C + ((size_t)m * L + l) * K * ds;", "C + ((size_t)m * L) * K * ds;"),
    "encode_plus_sign": ("float t = r[j] - cw[j];", "float t = r[j] + cw[j];"),
    "encode_subspace_offset": ("X[n * D + (int64_t)m * ds + j]", "X[n * D + (int64_t)m + j]"),
    "philox_lanes_swapped": ("c1 = lo1;", "c1 = lo0;"),
    "philox_key_schedule": ("k1 += 0xBB67AE8584CAA73Bull;", "k1 += 0x9E3779B97F4A7C15ull;"),
    "uniform_52_bits": ("(out[0] >> 11)", "(out[0] >> 12)"),
    "topk_last_tie": ("(best < 0 || y[v] > y[best])", "(best < 0 || y[v] >= y[best])"),
    "sample_ge": ("if (cum > t)", "if (cum >= t)"),
    "sample_no_temperature": ("(double)val[0]) / temperature);\n        if", "(double)val[0]));\n        if"),
}


def _checks(golden_dir):
    return [
        lambda: pins.check_bf16_golden(golden_dir),
        lambda: pins.check_pack10_golden(golden_dir),
        lambda: pins.check_decode_golden(golden_dir),
        pins.check_brute_force_tiny,
        pins.check_digit_encoded,
        pins.check_special_cases,
        pins.check_softcap,
        pins.check_argmax,
        lambda: pins.check_pages_fp32_identity(nrows=40),
        pins.check_encode_brute_force,
        pins.check_encode_vq,
        pins.check_encode_planted,
        pins.check_philox_numpy,
        pins.check_topk,
        pins.check_sampling,
    ]


def _build_mutant(name, tmp):
    old, new = MUTATIONS[name]
    text = open(SRC).read()
    assert old in text, name
    path = os.path.join(tmp, f"{name}.c")
    with open(path, "w") as f:
        f.write(text.replace(old, new))
    so = os.path.join(tmp, f"{name}.so")
    subprocess.check_call(["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fPIC",
                           "-shared", "-o", so, path, "-lm"])
    return so


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(name, golden_dir, monkeypatch, tmp_path):
    real = oracle._load()
    so = _build_mutant(name, str(tmp_path))
    lib = ctypes.CDLL(so)
    # give the mutant the same signatures as the real oracle
    for sym in ("rqo_lut_build_f64", "rqo_lut_build_f32", "rqo_logits_lut_f64",
                "rqo_logits_lut_f32", "rqo_logits_direct_f64", "rqo_logits_direct_f32",
                "rqo_softcap_f64", "rqo_argmax_f32", "rqo_argmax_f64",
                "rqo_f32_to_bf16_rne", "rqo_decode_rows_bf16", "rqo_packed10_row_bytes",
                "rqo_pack10", "rqo_unpack10", "rqo_encode_f32",
                "rqo_philox4x64_10", "rqo_uniform", "rqo_topk_f32", "rqo_sample_position"):
        src, dst = getattr(real, sym), getattr(lib, sym)
        dst.restype, dst.argtypes = src.restype, src.argtypes
    monkeypatch.setattr(oracle, "_lib", lib)
    failed = 0
    for chk in _checks(golden_dir):
        try:
            chk()
        except AssertionError:
            failed += 1
    assert failed > 0, f"mutation {name} went unnoticed by every pin"


def test_unmutated_oracle_passes_all_checks(golden_dir):
    for chk in _checks(golden_dir):
        chk()
