"""The oracle's pins catch plausible mistakes: each mutant below is a copy of
the oracle source with one planted error (built on the CPU in a temporary
directory), and at least one pin must fail against it."""
import os
import shutil

import pytest

import test_oracle_pins as pins

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(os.path.dirname(HERE), "oracle", "qlora_oracle.c")

# (name, original text, planted replacement)
MUTANTS = [
    ("ties_to_upper", "if (dj < bd) { bd = dj; best = j; }", "if (dj <= bd) { bd = dj; best = j; }"),
    ("nibble_order", "if ((i & 1) == 0) codes[i >> 1] |= (uint8_t)(c << 4);\n            else              codes[i >> 1] |= (uint8_t)c;",
     "if ((i & 1) == 1) codes[i >> 1] |= (uint8_t)(c << 4);\n            else              codes[i >> 1] |= (uint8_t)c;"),
    ("table_offset", "0.5 * (1.0 / 32.0 + 1.0 / 30.0)", "0.5 * (1.0 / 32.0 + 1.0 / 31.0)"),
    ("fwd_drops_scale", "Y[ii * N + n] = acc + s * lora;", "Y[ii * N + n] = acc + lora;"),
    ("fwd_transposed_B", "lora += u[j] * (double)bf16_to_f32(B[n * r + j]);",
     "lora += u[j] * (double)bf16_to_f32(B[(int64_t)j * N + n]);"),
    ("dx_drops_lora", "dX[ii * K + k] = acc[k] + s * lora;", "dX[ii * K + k] = acc[k];"),
    ("dB_uses_G", "acc[(n - n0) * r + j] += g * U[m * r + j];", "acc[(n - n0) * r + j] += g * G[m * r + j];"),
    ("dA_drops_scale", "dA[(int64_t)j * K + k] = s * acc[j * 64 + (k - k0)];", "dA[(int64_t)j * K + k] = acc[j * 64 + (k - k0)];"),
    ("offset_wrong_count", "(float)(sum / (double)nb)", "(float)(sum / (double)(nb + 1))"),
    ("dequant_offset_sign", "    return t + offset;", "    return t - offset;"),
    ("bf16_truncates", "uint32_t rounded = u + 0x7FFFu + lsb;", "uint32_t rounded = u + 0u * lsb;"),
    ("absmax_not_abs", "float av = fabsf(v);", "float av = v;"),
    ("t8_scale_128", "out[k] = (float)(k - 127) / 127.0f;", "out[k] = (float)(k - 127) / 128.0f;"),
    ("merge_ignores_sign", "(double)sign * s * acc;", "s * acc;"),
    ("merge_transposed_A", "* (double)bf16_to_f32(A[(int64_t)j * K + k]);\n            double v",
     "* (double)bf16_to_f32(A[k * r + j]);\n            double v"),
    ("adamw_no_bias_correction", "p[i] - lr * (m[i] / bc1)", "p[i] - lr * (m[i])"),
    ("adamw_coupled_decay", "p[i] = p[i] * (1.0 - lr * wd);", "g += wd * p[i];"),
    ("merge_rounds_down", "ldexp(nearbyint(ldexp(ax, -ulp_exp)), ulp_exp)", "ldexp(floor(ldexp(ax, -ulp_exp)), ulp_exp)"),
]

PINS = [
    pins.test_nf4_table_matches_library_quantiles,
    pins.test_nearest_ties_go_low,
    pins.test_q8_ties_go_low,
    pins.test_t8_table,
    pins.test_packing_golden,
    pins.test_roundtrip_lossless_without_dq,
    pins.test_equal_absmax_dq_is_lossless,
    pins.test_zero_and_partial_blocks,
    pins.test_error_bound,
    pins.test_dq_offset_is_mean,
    pins.test_dq_constant_error_bound,
    pins.test_fwd_vs_torch_linear,
    pins.test_bwd_vs_autograd,
    pins.test_zero_B_noop_and_zero_dA,
    pins.test_lora_merge_brute_force,
    pins.test_adamw_vs_torch_optim,
]


@pytest.fixture(scope="module")
def mutant_dir(tmp_path_factory):
    return tmp_path_factory.mktemp("oracle_mutants")


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(O, mutant_dir, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    path = os.path.join(mutant_dir, f"{name}.c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    lib = O.build(force=True, src=path, out=os.path.join(mutant_dir, f"lib{name}.so"))
    caught = []
    O.use_library(lib)
    try:
        for pin in PINS:
            try:
                pin(O)
            except AssertionError:
                caught.append(pin.__name__)
    finally:
        O.use_library(O.build())
    assert caught, f"no pin fails for mutant {name}"
