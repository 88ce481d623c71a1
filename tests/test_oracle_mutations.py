"""Negative controls for the oracle's pins.

Each case plants one plausible mistake in a copy of oracle/orc.c (on the CPU,
in a temporary directory), builds it, and checks that at least one pin of
tests/oracle_pins.py catches it.  A pin set that lets a planted mistake
through is too weak to vouch for the oracle.
"""
import os

import pytest

import oracle
from oracle.build import SRC, build_oracle
from tests import oracle_pins

MUTANTS = [
    ("nibble_order", "packed[i] = (uint8_t)(c0 | (c1 << 4));",
     "packed[i] = (uint8_t)(c1 | (c0 << 4));"),
    ("mx_emax_off_by_one", "int e = (e2 - 1) - 2;", "int e = (e2 - 1) - 1;"),
    ("eps_outside_sqrt", "return 1.0 / sqrt(ss / (double)n + (double)eps);",
     "return 1.0 / (sqrt(ss / (double)n) + (double)eps);"),
    ("mean_over_n_minus_1", "return 1.0 / sqrt(ss / (double)n + (double)eps);",
     "return 1.0 / sqrt(ss / (double)(n - 1) + (double)eps);"),
    ("residual_dropped", "s = s + elem_to_float(io, residual[m * H + j]);",
     "s = s + 0.0f * elem_to_float(io, residual[m * H + j]);"),
    ("partials_in_fp64", "float s = elem_to_float(io, parts[0][m * H + j]);",
     "double s = elem_to_float(io, parts[0][m * H + j]);"),
    ("plain_weight_in_gemma", "(1.0 + orc_bf16_to_double(w[d]))", "orc_bf16_to_double(w[d])"),
    ("ties_away_from_zero", "double n = nearbyint(fabs(v) / quantum);",
     "double n = round(fabs(v) / quantum);"),
    ("reciprocal_multiply", "float t = elem_to_float(io, y[j]) / scale;",
     "float t = elem_to_float(io, y[j]) * (1.0f / scale);"),
    ("fp8_max_240", "amax / 448.0f", "amax / 240.0f"),
    ("e4m3_no_subnormals", "round_to_grid(v, 3, -6)", "round_to_grid(v, 3, -7)"),
    ("q_from_gate_slot", "gemma_norm_head(row + (int64_t)2 * h * D, q_weight",
     "gemma_norm_head(row + (int64_t)(2 * h + 1) * D, q_weight"),
    ("k_offset_without_gates", "row + (int64_t)2 * Hq * D + (int64_t)h * D, k_weight",
     "row + (int64_t)Hq * D + (int64_t)h * D, k_weight"),
    ("zero_group_scale_zero", "float scale = (amax == 0.0f) ? 1.0f : amax / 448.0f;",
     "float scale = (amax == 0.0f) ? 0.0f : amax / 448.0f;"),
    ("weight_applied_twice",
     "ybuf[j] = elem_from_double(io, elem_to_double(io, hbuf[j]) * rstd *",
     "ybuf[j] = elem_from_double(io, elem_to_double(io, weight[j]) * elem_to_double(io, hbuf[j]) * rstd *"),
    # binary16 input/output
    ("fp16_nine_mantissa_bits", "round_to_grid(v, 10, -14)", "round_to_grid(v, 9, -14)"),
    ("fp16_no_subnormal_grid", "round_to_grid(v, 10, -14)", "round_to_grid(v, 10, -15)"),
    ("fp16_overflow_saturates", "return (uint16_t)(sign | 0x7C00u);",
     "return (uint16_t)(sign | 0x7BFFu);"),
    ("fp16_decode_bias", "mag = ldexp(1024.0 + m, e - 25);", "mag = ldexp(1024.0 + m, e - 24);"),
    ("fp16_weight_read_as_bf16", "elem_to_double(io, weight[j]));",
     "orc_bf16_to_double(weight[j]));"),
    ("fp16_quant_reads_bf16", "float t = elem_to_float(io, y[j]) / scale;",
     "float t = elem_to_float(ORC_IO_BF16, y[j]) / scale;"),
    ("fp16_h_rounded_as_bf16", "hbuf[j] = elem_from_double(io, (double)s);",
     "hbuf[j] = orc_bf16_from_double((double)s);"),
    # hc_mix (reading A19)
    ("hc_gate_sign", "g[e] = 1.0 / (1.0 + exp(-z));", "g[e] = 1.0 / (1.0 + exp(z));"),
    ("hc_gate_tanh", "g[e] = 1.0 / (1.0 + exp(-z));", "g[e] = 0.5 * (1.0 + tanh(z));"),
    ("hc_streams_interleaved", "u += g[(int64_t)s * C + c] * orc_bf16_to_double(xr[(int64_t)s * C + c]);",
     "u += g[(int64_t)c * hc + s] * orc_bf16_to_double(xr[(int64_t)c * hc + s]);"),
    ("hc_gate_applied_to_stream0", "orc_bf16_to_double(xr[(int64_t)s * C + c]);",
     "orc_bf16_to_double(xr[c]);"),
    ("hc_w_down_transposed", "orc_bf16_to_double(w_down[(int64_t)j * K + k]);",
     "orc_bf16_to_double(w_down[k * r + j]);"),
    ("hc_w_up_transposed", "z += t[j] * orc_bf16_to_double(w_up[e * r + j]);",
     "z += t[j] * orc_bf16_to_double(w_up[(int64_t)j * K + e]);"),
    ("hc_last_stream_dropped", "for (int s = 0; s < hc; ++s)", "for (int s = 0; s < hc - 1; ++s)"),
    ("hc_t_rounded_to_bf16", "t[j] = acc;", "t[j] = orc_bf16_to_double(orc_bf16_from_double(acc));"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} missing"
    mut_src = os.path.join(tmp_path, "orc_mut.c")
    with open(mut_src, "w") as fh:
        fh.write(src.replace(old, new))
    lib_path = build_oracle(src=mut_src, out=os.path.join(tmp_path, "liborc_mut.so"),
                            extra_flags=("-Wno-error",), force=True)
    lib = oracle.load(lib_path)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(lib)
        except (AssertionError, oracle.OracleError) as e:
            caught.append((pin.__name__, str(e)[:80]))
            break
    assert caught, f"no pin caught the planted mistake {name}"
