"""The pins must catch plausible mistakes.  Each case copies ``oracle.c``,
plants one mistake in the copy (on the CPU, in a temporary directory), builds
it and checks that a pin from the other test files now fails."""
from __future__ import annotations

import os

import pytest

import oracle
import test_oracle_a8 as a8
import test_oracle_codecs as codecs
import test_oracle_linear as lin
import test_oracle_lora as lora
import test_oracle_quant as quant
import test_oracle_swiglu as swiglu

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

# (name, original text, planted text, pin that must now fail)
MUTANTS = [
    ("nibble order swapped",
     "return (k & 1) ? (b >> 4) : (b & 15);",
     "return (k & 1) ? (b & 15) : (b >> 4);",
     lambda o: lin.test_integer_special_case(o, "int4_sym", 64)),
    ("zero-point added instead of subtracted",
     "return (float)(q - z) * s;",
     "return (float)(q + z) * s;",
     lambda o: lin.test_integer_special_case(o, "int4_asym", 32)),
    ("bias dropped",
     "      if (bias) acc += (double)orc_bf16_to_f32(bias[n]);\n      if (y64) y64[m * N + n]",
     "      if (y64) y64[m * N + n]",
     lambda o: lin.test_linear_matches_exact_rational(o, 16)),
    ("reduction index reversed",
     "acc += (double)orc_bf16_to_f32(xr[k]) * (double)w[k];",
     "acc += (double)orc_bf16_to_f32(xr[k]) * (double)w[K - 1 - k];",
     lambda o: lin.test_integer_special_case(o, "int8_sym", 128)),
    ("bf16 ties rounded away from zero",
     "double r = nearbyint(a / quantum) * quantum;",
     "double r = round(a / quantum) * quantum;",
     lambda o: codecs.test_bf16_from_f32_matches_torch(o)),
    ("E4M3 exponent bias off by one",
     "else v = ldexp(1.0 + m / 8.0, e - 7);",
     "else v = ldexp(1.0 + m / 8.0, e - 8);",
     lambda o: codecs.test_e4m3_values_match_torch(o)),
    ("NVFP4 tensor scale missing the 6",
     "float ts = (float)(amax / (6.0 * 448.0));",
     "float ts = (float)(amax / 448.0);",
     lambda o: quant.test_nvfp4_properties(o)),
    ("MXFP4 shared exponent without the E2M1 maximum exponent",
     "int se = (ex - 1) - 2;",
     "int se = (ex - 1);",
     lambda o: quant.test_mxfp4_properties(o)),
    ("INT scale divided by qmax+1",
     "uint16_t sb = orc_f64_to_bf16(amax / (double)qmax);",
     "uint16_t sb = orc_f64_to_bf16(amax / (double)(qmax + 1));",
     lambda o: quant.test_sym_properties(o, "int8_sym", 127, 64)),
    ("asym zero-point sign flipped",
     "double zr = nearbyint(-lo / s);",
     "double zr = nearbyint(lo / s);",
     lambda o: quant.test_asym_properties(o, 128)),
    ("codebook norm not divided by sqrt(K)",
     "double norm64 = sqrt(ss) / sqrt((double)K);",
     "double norm64 = sqrt(ss);",
     lambda o: quant.test_cb4_nearest_neighbour(o)),
    ("Lloyd-Max level uses the wrong cell edge",
     "double nc = (normal_pdf(t[i]) - normal_pdf(t[i + 1])) / p;",
     "double nc = (normal_pdf(t[i]) - normal_pdf(t[i + 1])) / p * 1.001;",
     lambda o: quant.test_lloyd_max_invariants(o)),
    ("FP8 sign dropped",
     "if (r < 0.0 && q != 0) q |= 0x80;",
     "if (r < 0.0 && q == 0) q |= 0x80;",
     lambda o: quant.test_fp8_properties(o, 32, "fp8_e4m3")),
    ("FP8 scale from the wrong maximum",
     "const double fmax_code = e5m2 ? 57344.0 : 448.0;",
     "const double fmax_code = e5m2 ? 57344.0 : 240.0;",
     lambda o: quant.test_fp8_properties(o, 128, "fp8_e4m3")),
    ("E5M2 exponent bias off by one",
     "else v = ldexp(1.0 + m / 4.0, e - 15);",
     "else v = ldexp(1.0 + m / 4.0, e - 16);",
     lambda o: codecs.test_e5m2_values_match_torch(o)),
    ("SwiGLU reads the gate half as up",
     "double up = (double)orc_bf16_to_f32(x2[m * 2 * K + k]);",
     "double up = (double)orc_bf16_to_f32(x2[m * 2 * K + K + k]);",
     lambda o: swiglu.test_swiglu_layout_and_rounding(o)),
    ("INT2 field order reversed in the dequant",
     "int c = (((const uint8_t*)codes)[n * (K / 4) + k / 4] >> (2 * (k & 3))) & 3;",
     "int c = (((const uint8_t*)codes)[n * (K / 4) + k / 4] >> (6 - 2 * (k & 3))) & 3;",
     lambda o: lin.test_integer_special_case(o, "int2_sym", 64)),
    ("stochastic requantization compares the wrong way",
     "q = f + (u < t - f ? 1.0 : 0.0);",
     "q = f + (u > t - f ? 1.0 : 0.0);",
     lambda o: lora.test_stochastic_rounding_is_unbiased(o)),
    ("activation scale from 128 instead of 127",
     "float s = (float)(amax / 127.0);",
     "float s = (float)(amax / 128.0);",
     lambda o: a8.test_activation_scale_and_error_bound(o)),
    ("INT3 bit stream read most-significant bit first",
     "for (int b = 0; b < 3; ++b) c |= ((row[(3 * k + b) >> 3] >> ((3 * k + b) & 7)) & 1) << b;",
     "for (int b = 0; b < 3; ++b) c |= ((row[(3 * k + b) >> 3] >> (7 - ((3 * k + b) & 7))) & 1) << b;",
     lambda o: lin.test_integer_special_case(o, "int3_sym", 32)),
    ("E2M1 tie broken toward the odd code",
     "if (a == mid) { code = (i % 2 == 0) ? i : i + 1; break; }",
     "if (a == mid) { code = (i % 2 == 0) ? i + 1 : i; break; }",
     lambda o: codecs.test_e2m1_ties_and_saturation(o)),
]


@pytest.mark.parametrize("name,orig,planted,pin", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pin_catches_planted_mistake(tmp_path, name, orig, planted, pin):
    text = open(SRC).read()
    assert text.count(orig) == 1, f"mutation site for '{name}' not found exactly once"
    src = tmp_path / "oracle_mutant.c"
    src.write_text(text.replace(orig, planted))
    # a distinct file name per mutant: the dynamic loader may hand back an
    # already-loaded library when a new file reuses an old one's identity
    tag = "".join(ch for ch in name if ch.isalnum())
    so = oracle.build(force=True, out_path=str(tmp_path / f"liboracle_{tag}.so"), src=str(src))
    mutant = oracle.Oracle(oracle.load(so))
    with pytest.raises(AssertionError):
        pin(mutant)
