"""Planted mistakes: the oracle's pins must reject a wrong oracle (CPU only).

Each case copies the oracle's C source, plants one plausible mistake in the copy (a flipped tie
rule, a dropped factor, a wrong sign, a swapped nibble, an off-by-one...), builds it with the
same flags, loads it in place of the real oracle and runs the pins that cover that part of the
method.  At least one pin must fail for every mutant; the unmodified source, built the same
way, must pass all of them.  Nothing here runs on a GPU or touches the CUDA library.
"""
import os
import subprocess

import pytest

import oracle

from . import test_oracle_codebooks as PC
from . import test_oracle_nested as PN
from . import test_oracle_quantize as PQ
from . import test_oracle_step as PS

SRC = os.path.join(os.path.dirname(oracle.__file__), "bnbq_oracle.c")


def _codebook_pins(o):
    return [lambda: PC.test_unsigned_dynamic_structure(o), lambda: PC.test_signed_dynamic_structure(o),
            lambda: PC.test_dynamic_codes_correctly_rounded(o), lambda: PC.test_nf4_normal_quantiles(o),
            lambda: PC.test_fp4_e2m1_values(o), lambda: PC.test_linear_code(o)]


def _quantize_pins(o):
    return [lambda: PQ.test_nearest_code_exact_bruteforce(o, "signed"),
            lambda: PQ.test_nearest_code_exact_bruteforce(o, "nf4"),
            lambda: PQ.test_quantize_blockwise_matches_bruteforce(o, "signed", 256, False),
            lambda: PQ.test_quantize_blockwise_matches_bruteforce(o, "nf4", 64, True),
            lambda: PQ.test_normalisation_is_the_correctly_rounded_quotient(o),
            lambda: PQ.test_round_trip_every_code(o, "signed"),
            lambda: PQ.test_nf4_nibble_order(o),
            lambda: PQ.test_dequantize_bf16_matches_torch_rounding(o),
            lambda: PQ.test_dequantize_bf16_ties_to_even(o),
            lambda: PQ.test_error_bound(o, "signed")]


def _step_pins(o):
    return [lambda: PS.test_adamw_32bit_matches_torch(o, 0.01), lambda: PS.test_adamw_first_step_closed_form(o),
            lambda: PS.test_adam_l2_matches_torch(o), lambda: PS.test_momentum_matches_torch_sgd(o, 0.01),
            lambda: PS.test_momentum_first_step(o), lambda: PS.test_lion_sign_update(o),
            lambda: PS.test_lion_decay_uses_the_old_parameter(o),
            lambda: PS.test_rmsprop_matches_torch(o, 0.01), lambda: PS.test_rmsprop_first_step_closed_form(o),
            lambda: PS.test_rmsprop_8bit_step_matches_torch(o), lambda: PS.test_8bit_first_step_equals_32bit(o),
            lambda: PS.test_8bit_step_from_quantized_state_matches_torch(o),
            lambda: PS.test_zero_gradient_zero_state_stays(o), lambda: PS.test_bf16_gradients_are_widened_exactly(o)]


def _nested_pins(o):
    return [lambda: PN.test_offset_is_the_correctly_rounded_mean(o, 4097),
            lambda: PN.test_equal_scales_rebuild_exactly(o), lambda: PN.test_two_scales_map_to_the_ends_of_the_code(o),
            lambda: PN.test_rebuild_error_within_half_the_code_gap(o, 4096 + 513)]


PINS = {"codebooks": _codebook_pins, "quantize": _quantize_pins, "step": _step_pins, "nested": _nested_pins}

# name: (area, [(text in the source, planted replacement), ...])
MUTANTS = {
    "tie goes to the upper code": ("quantize", [("if (xn > oracle_code_mid(code, j)) q++;",
                                                 "if (xn >= oracle_code_mid(code, j)) q++;")]),
    "block absmax skips the last element": ("quantize", [("    for (int64_t i = 0; i < len; i++) {\n        float m = fabsf(v[i]);",
                                                          "    for (int64_t i = 0; i + 1 < len; i++) {\n        float m = fabsf(v[i]);")]),
    "4-bit nibbles swapped": ("quantize", [("(uint8_t)(out[e >> 1] | (q << 4)); /* even", "(uint8_t)(out[e >> 1] | q); /* even"),
                                           ("(uint8_t)(out[e >> 1] | q);        /* odd", "(uint8_t)(out[e >> 1] | (q << 4)); /* odd")]),
    "dequantize uses the first block's scale": ("quantize", [("float v = code[idx] * absmax[e / B];",
                                                              "float v = code[idx] * absmax[0];")]),
    "bf16 narrowing truncates": ("quantize", [("u += 0x7fffu + lsb;", "u += 0u * lsb;")]),
    "dynamic code on the lower bin edge": ("codebooks", [("(double)((1 << nE) + 9 * (k + 1))", "(double)((1 << nE) + 9 * k)")]),
    "NF4 offset delta = 1/30": ("codebooks", [("const double delta = 0.5 * (1.0 / 30.0 + 1.0 / 32.0);",
                                               "const double delta = 1.0 / 30.0;")]),
    "NF4 negative half spaced like the positive half": ("codebooks", [(
        "double prob = delta + (0.5 - delta) * (double)k / 7.0;", "double prob = delta + (0.5 - delta) * (double)k / 8.0;")]),
    "NF4 positive half not scaled to 1": ("codebooks", [(
        "double prob = 0.5 + (0.5 - delta) * (double)k / 8.0;\n        out[c++] = (float)(normal_quantile(prob) / scale);",
        "double prob = 0.5 + (0.5 - delta) * (double)k / 8.0;\n        out[c++] = (float)(normal_quantile(prob));")]),
    "FP4 exponent without its bias": ("codebooks", [("ldexp(1.0 + 0.5 * (double)f, e - 1)", "ldexp(1.0 + 0.5 * (double)f, e)")]),
    "linear code steps by 2/256": ("codebooks", [("(float)(-1.0 + 2.0 * (double)k / 255.0)", "(float)(-1.0 + 2.0 * (double)k / 256.0)")]),
    "FP4 spare pattern duplicates a code": ("codebooks", [("out[c++] = (float)(0.25 / 6.0);", "out[c++] = (float)(0.5 / 6.0);")]),
    "Adam m drops (1 - b1)": ("step", [("float m1 = d->b1 * (*m) + d->omb1 * g;", "float m1 = d->b1 * (*m) + g;")]),
    "Adam v not squared": ("step", [("float v1 = d->b2 * (*v) + (d->omb2 * g) * g;", "float v1 = d->b2 * (*v) + (d->omb2 * g);")]),
    "decoupled decay with the wrong sign": ("step", [("(float)(1.0 - (double)hp->lr * (double)hp->weight_decay)",
                                                      "(float)(1.0 + (double)hp->lr * (double)hp->weight_decay)")]),
    "no first-moment bias correction": ("step", [("d.step_size = (float)((double)hp->lr / (1.0 - pow(b1, (double)t)));",
                                                  "d.step_size = hp->lr;")]),
    "second-moment correction multiplied": ("step", [("float denom = sqrtf(v1) / d->sqrt_bc2 + d->eps;",
                                                      "float denom = sqrtf(v1) * d->sqrt_bc2 + d->eps;")]),
    "Lion sign flipped": ("step", [("float s = (c > 0.0f) ? 1.0f : ((c < 0.0f) ? -1.0f : 0.0f);",
                                    "float s = (c > 0.0f) ? -1.0f : ((c < 0.0f) ? 1.0f : 0.0f);")]),
    "momentum with dampening": ("step", [("float m1 = d->b1 * (*m) + g;", "float m1 = d->b1 * (*m) + d->omb1 * g;")]),
    "RMSprop eps inside the root": ("step", [("float denom = sqrtf(v1) + d->eps;", "float denom = sqrtf(v1 + d->eps);")]),
    "bf16 narrowing rounds ties up": ("quantize", [("u += 0x7fffu + lsb;", "u += 0x8000u + 0u * lsb;")]),
    "block absmax of signed values": ("quantize", [("float m = fabsf(v[i]);", "float m = v[i];")]),
    "step leaves the last element of a ragged block": ("step", [(
        "int64_t len = (n - start < B) ? (n - start) : B;\n        /* 1. load",
        "int64_t len = (n - start < B) ? (n - start - 1) : B;\n        /* 1. load")]),
    "normalisation by a rounded reciprocal": ("quantize", [("float xn = (absmax == 0.0f) ? 0.0f : x / absmax;",
                                                            "float xn = (absmax == 0.0f) ? 0.0f : x * (1.0f / absmax);")]),
    "requantize with the old block scale": ("step", [("float a1 = block_absmax(mbuf, len);\n            absmax1[b] = a1;",
                                                      "float a1 = absmax1[b];")]),
    "state dequantized with the next block's scale": ("step", [("mbuf[i] = code1[((const uint8_t*)s1)[e]] * absmax1[b];",
                                                                "mbuf[i] = code1[((const uint8_t*)s1)[e]] * absmax1[(b + 1 < nb) ? b + 1 : b];")]),
    "Lion state becomes the interpolation c": ("step", [("*m = d->b2 * (*m) + d->omb2 * g;", "*m = c;")]),
    "Lion decay applied after the sign step": ("step", [("pv = pv * d->decay;\n        pv = pv - d->lr * s;",
                                                         "pv = pv - d->lr * s;\n        pv = pv * d->decay;")]),
    "second-moment correction uses beta1": ("step", [("d.sqrt_bc2 = (float)sqrt(1.0 - pow(b2, (double)t));",
                                                      "d.sqrt_bc2 = (float)sqrt(1.0 - pow(b1, (double)t));")]),
    "bf16 widening drops the sign": ("step", [("uint32_t u = (uint32_t)h << 16;", "uint32_t u = (uint32_t)(h & 0x7fffu) << 16;")]),
    "RMSprop alpha and 1 - alpha swapped": ("step", [("float v1 = d->b1 * (*m) + (d->omb1 * g) * g;",
                                                      "float v1 = d->omb1 * (*m) + (d->b1 * g) * g;")]),
    "nested mean divides by nb + 1": ("nested", [("return (float)(total / (double)nb);", "return (float)(total / (double)(nb + 1));")]),
    "nested mean accumulated in binary32": ("nested", [("        double s = 0.0;", "        float s = 0.0f;")]),
    "nested offset not stored": ("nested", [("    *offset = mean;", "    *offset = 0.0f;")]),
    "nested scales not centred": ("nested", [("centred[i] = absmax[i] - mean;", "centred[i] = absmax[i];")]),
    "nested rebuild adds before multiplying": ("nested", [("out[i] = code2[qabs[i]] * absmax2[i / ORACLE_NEST_B] + offset;",
                                                          "out[i] = (code2[qabs[i]] + offset) * absmax2[i / ORACLE_NEST_B];")]),
}


def _build(tmp_path, name, edits):
    src = open(SRC).read()
    for old, new in edits:
        assert src.count(old) == 1, f"{name}: the planted text must occur exactly once: {old!r}"
        src = src.replace(old, new)
    d = tmp_path / "src"
    d.mkdir()
    c = d / "bnbq_oracle.c"
    c.write_text(src)
    for h in ("bnbq_oracle.h",):
        (d / h).write_text(open(os.path.join(os.path.dirname(SRC), h)).read())
    so = tmp_path / "liboracle_mutant.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math", "-o",
                    str(so), str(c), "-lm"], check=True)
    return str(so)


def _failures(path, area):
    prev = oracle.swap_library(path)
    failed = 0
    try:
        for pin in PINS[area](oracle):
            try:
                pin()
            except Exception:  # an assertion, or a rejected argument
                failed += 1
    finally:
        oracle.restore_library(prev)
    return failed


@pytest.mark.parametrize("area", sorted(PINS))
def test_unmodified_source_passes_the_pins(tmp_path, area):
    assert _failures(_build(tmp_path, "unmodified", []), area) == 0


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(tmp_path, name):
    area, edits = MUTANTS[name]
    assert _failures(_build(tmp_path, name, edits), area) > 0, f"no pin rejects the mutant '{name}'"
