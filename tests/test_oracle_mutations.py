"""Plants plausible mistakes in a temporary copy of the oracle (CPU only) and
checks that the pins in test_oracle_pins.py catch each one.

Every mutant is a one-token edit of oracle.c: a wrong rounding mode, a wrong
constant, a transposed or shifted index, a dropped term, a scale applied the
wrong way round, a wrong bit position or code.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

# (name, original text, mutated text, pins expected to catch it)
MUTANTS = [
    ("round_half_away_ternarize", "float v = rintf(r);", "float v = roundf(r);",
     [pins.test_ternarize_golden]),
    ("quant_scale_128", "float sc = 127.0f / den;", "float sc = 128.0f / den;",
     [pins.test_quant_golden, pins.test_quant_invariants]),
    ("quant_round_half_away", "float r = rintf(v);", "float r = roundf(v);",
     [pins.test_quant_golden]),
    ("gemm_transposed_index", "const int8_t *wr = Wt + n * K;", "const int8_t *wr = Wt + m * K;",
     [lambda o: pins.test_gemm_bruteforce(o, 2, 3, 67), pins.test_gemm_special_weights]),
    ("gemm_dropped_last_term",
     "for (int64_t k = 0; k < K; ++k)\n            acc += (int64_t)qr[k] * (int64_t)wr[k];\n        if (acc",
     "for (int64_t k = 0; k < K - 1; ++k)\n            acc += (int64_t)qr[k] * (int64_t)wr[k];\n        if (acc",
     [lambda o: pins.test_gemm_bruteforce(o, 1, 5, 7)]),
    ("rescale_scale_inverted", "* (double)gamma / (double)s[m];", "* (double)gamma * (double)s[m];",
     [pins.test_rescale_closed_form, pins.test_bitlinear_within_quantisation_error]),
    ("absmean_sum_not_mean", "return (float)(sum / ((double)N * (double)K));", "return (float)(sum / (double)K);",
     [pins.test_ternarize_golden, pins.test_absmean_matches_library_mean]),
    ("device_layout_wrong_shift", "int shift = 2 * (int)((k % 16) / 4);\n            row[byte]",
     "int shift = 2 * (int)(k % 4);\n            row[byte]",
     [pins.test_device_pack_golden]),
    ("device_code_negated", "code = (unsigned)(w + 1);\n                else",
     "code = (unsigned)(1 - w);\n                else",
     [pins.test_device_pack_golden, pins.test_code_mapping_golden]),
    ("ternarize_no_clamp", "if (v > 1.0f) v = 1.0f;", "if (v > 2.0f) v = 2.0f;",
     [pins.test_ternarize_golden, pins.test_ternarize_invariants]),
]


@pytest.fixture
def mutant_lib(tmp_path):
    saved = oracle._lib()

    def build(orig, new):
        src = open(SRC, encoding="utf-8").read()
        assert src.count(orig) == 1, orig
        path = tmp_path / "mutant.c"
        path.write_text(src.replace(orig, new), encoding="utf-8")
        so = tmp_path / f"libmutant_{abs(hash(new))}.so"
        subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                        "-ffp-contract=off", "-o", str(so), str(path), "-lm"], check=True)
        lib = ctypes.CDLL(str(so))
        # reuse the signatures of the real library
        for name in ("oracle_absmean", "oracle_ternarize", "oracle_quant_act", "oracle_gemm_i32",
                     "oracle_gemm_i32_sampled", "oracle_rescale", "oracle_bitlinear",
                     "oracle_canonical_packed_bytes", "oracle_pack_canonical",
                     "oracle_unpack_canonical", "oracle_device_packed_bytes",
                     "oracle_pack_device", "oracle_unpack_device"):
            f, g = getattr(lib, name), getattr(saved, name)
            f.restype, f.argtypes = g.restype, g.argtypes
        oracle._LIB = lib

    yield build
    oracle._LIB = saved


@pytest.mark.parametrize("name,orig,new,catchers", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(mutant_lib, name, orig, new, catchers):
    mutant_lib(orig, new)
    caught = 0
    for check in catchers:
        try:
            check(oracle)
        except (AssertionError, OverflowError):
            caught += 1
    assert caught >= 1, f"no pin caught mutant {name}"
