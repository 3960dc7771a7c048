"""Plant plausible mistakes in copies of the oracle and check that a pin catches each.

Each mutant is the oracle source with one textual change (a wrong exponent
bias, a dropped term, a swapped nibble order, a wrong sign, a transposed
index ...). It is compiled on the CPU into a temporary library, swapped in,
and every pin is run; at least one pin must fail. Mutations are chosen so the
broken oracle never reads outside its buffers.
"""
import os
import subprocess

import pytest

import oracle
import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "qmm_oracle.c")

MUTANTS = [
    ("fp16_exponent_bias", "e - 25);", "e - 24);"),
    ("fp16_subnormal_scale", "ldexp((double)m, -24);", "ldexp((double)m, -23);"),
    ("fp16_implicit_bit", "(double)(m | 0x400)", "(double)(m)"),
    ("bf16_exponent_bias", "e - 134);", "e - 135);"),
    ("bf16_subnormal_scale", "ldexp((double)m, -133);", "ldexp((double)m, -134);"),
    ("q8_unsigned_codes", "(double)(int8_t)qs[j] * d", "(double)(uint8_t)qs[j] * d"),
    ("q4_offset", "(int)(qs[j] & 0x0f) - 8)", "(int)(qs[j] & 0x0f) - 7)"),
    ("q4_nibble_order", "w[j] = (double)((int)(qs[j] & 0x0f) - 8) * d;\n      w[j + 16] = (double)((int)(qs[j] >> 4) - 8) * d;",
     "w[j + 16] = (double)((int)(qs[j] & 0x0f) - 8) * d;\n      w[j] = (double)((int)(qs[j] >> 4) - 8) * d;"),
    ("scale_byte_order", "(uint16_t)(blk[0] | (blk[1] << 8));\n  double d", "(uint16_t)(blk[1] | (blk[0] << 8));\n  double d"),
    ("gemv_block_reversed", "ora_decode_block(wtype, W + (n * kb + b) * bb, w);\n        for (int j = 0; j < ORA_BLOCK; ++j) {\n          double p = w[j] * (double)X",
     "ora_decode_block(wtype, W + (n * kb + (kb - 1 - b)) * bb, w);\n        for (int j = 0; j < ORA_BLOCK; ++j) {\n          double p = w[j] * (double)X"),
    ("gemv_x_block_offset_dropped", "(double)X[m * K + b * ORA_BLOCK + j];", "(double)X[m * K + j];"),
    ("gemv_norm_signed", "acc += p;\n          nrm += fabs(p);\n        }\n      }\n      Y[(m - m0) * wn + (n - n0)] = acc;\n      if (S) S[(m - m0) * wn + (n - n0)] = nrm;\n    }\n  }\n}",
     "acc += p;\n          nrm += p;\n        }\n      }\n      Y[(m - m0) * wn + (n - n0)] = acc;\n      if (S) S[(m - m0) * wn + (n - n0)] = nrm;\n    }\n  }\n}"),
    ("quant_divisor_128", "amax / 127.0f", "amax / 128.0f"),
    ("quant_half_even", "roundf(v);", "rintf(v);"),
    ("quant_truncate", "roundf(v);", "truncf(v);"),
    ("quant_amax_signed", "float a = fabsf(x[j]);", "float a = x[j];"),
    ("q8q8_unsigned_weight", "s += (int64_t)(int8_t)blk[2 + j] * (int64_t)QX", "s += (int64_t)(uint8_t)blk[2 + j] * (int64_t)QX"),
    ("q8q8_dx_dropped", "acc += dw * dx * (double)s;", "acc += dw * (double)s;"),
    ("q8q8_gemv_unsigned_weight", "int64_t p = (int64_t)(int8_t)blk[2 + j]", "int64_t p = (int64_t)(uint8_t)blk[2 + j]"),
    ("silu_sign", "g / (1.0 + exp(-g)) * U[i]", "g / (1.0 + exp(g)) * U[i]"),
    ("swiglu_gate_up_swapped", "OUT[i] = g / (1.0 + exp(-g)) * U[i];", "OUT[i] = U[i] / (1.0 + exp(-U[i])) * g;"),
    ("prefill_wrong_decoder", "ora_bf16_to_double(Xbf[", "ora_half_to_double(Xbf["),
    ("half_round_half_up", "(rem == 0.5 && fmod(r, 2.0) != 0.0)", "(rem == 0.5)"),
    ("half_subnormal_spacing", "if (exp16 < -14) exp16 = -14;", "if (exp16 < -15) exp16 = -15;"),
    ("q8_0_codes_scaled_by_d", "const float v = x[j] * id;", "const float v = x[j] * d;"),
    ("q8_0_scale_byte_order", "blk[0] = (uint8_t)(h & 0xff);\n      blk[1] = (uint8_t)(h >> 8);",
     "blk[1] = (uint8_t)(h & 0xff);\n      blk[0] = (uint8_t)(h >> 8);"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, old, new, tmp_path):
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    mutated = src.replace(old, new, 1)
    assert mutated != src
    c_path = tmp_path / "mutant.c"
    so_path = tmp_path / "libmutant.so"
    c_path.write_text(mutated)
    subprocess.check_call(["gcc", *oracle._CFLAGS, str(c_path), "-o", str(so_path), "-lm"])
    failed = []
    oracle._swap_library(str(so_path))
    try:
        for pin in oracle_pins.PINS:
            try:
                pin()
            except AssertionError:
                failed.append(pin.__name__)
    finally:
        oracle._swap_library(None)
    assert failed, f"mutant {name} passed every pin"
