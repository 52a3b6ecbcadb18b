"""The oracle's pins must catch plausible mistakes.

Each case below plants one mistake in a copy of oracle/sbsa_oracle.c (a text edit,
compiled with gcc into a temporary library, on the CPU), swaps it in for the real
oracle, and runs every pin in test_oracle_pins.py.  At least one pin must fail for
each mutant; the real oracle passes them all.  The Python-side oracle functions (the
Light-Ulysses exchanges) get the same treatment: a mutated copy of one function is
swapped in for the pins' run.
"""
import ctypes
import inspect
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "sbsa_oracle.c")

MUTANTS = {
    # pool divides by the block size instead of the number of valid tokens
    "pool_divides_by_block": ("s / (double)(t1 - t0)", "s / (double)blk"),
    # pool also averages the padded tokens
    "pool_counts_padding": ("int t1 = t0 + blk < L ? t0 + blk : L;", "int t1 = t0 + blk;"),
    # score uses a transposed operand (key block i against query block j)
    "score_transposed": ("qmean_bh[(size_t)i * d + c] * kmean_bh[(size_t)j * d + c]",
                         "qmean_bh[(size_t)j * d + c] * kmean_bh[(size_t)i * d + c]"),
    # ties broken toward the higher block index
    "ties_to_higher_index": ("return (a->j > b->j) - (a->j < b->j);",
                             "return (a->j < b->j) - (a->j > b->j);"),
    # the diagonal competes like any other block instead of being forced
    "diagonal_not_forced": ("if (j != i) { cand[n].s", "if (1) { cand[n].s"),
    # attention forgets to mask padded keys
    "padded_keys_kept": ("if (u >= L) continue;\n            size_t krow", "size_t krow"),
    # softmax without the max subtraction
    "no_max_subtraction": ("double p = exp(logit[n] - m);", "double p = exp(logit[n]);"),
    # off-by-one in the gather of the kept block's tokens
    "gather_off_by_one": ("int u = cols[n / blk] * blk + n % blk;\n            logit[n]",
                          "int u = cols[n / blk] * blk + (n + 1) % blk;\n            logit[n]"),
    # the scale is dropped
    "scale_dropped": ("logit[n] = s * scale;", "logit[n] = s;"),
    # RoPE turns the wrong way round in the second component (a reflection, norms kept)
    "rope_sin_sign": ("out[(size_t)r * d + 2 * p + 1] = a * sn + b * c;",
                      "out[(size_t)r * d + 2 * p + 1] = -a * sn + b * c;"),
    # RoPE pairs of the row and column axes swapped
    "rope_axes_swapped": ("int axis = p < pt ? 0 : (p < pt + ph ? 1 : 2);",
                          "int axis = p < pt ? 0 : (p < pt + ph ? 2 : 1);"),
    # RoPE frequency exponent off by one pair
    "rope_freq_off_by_one": ("pow(theta, -(double)q / (double)np)", "pow(theta, -(double)(q + 1) / (double)np)"),
    # RoPE row index taken with the wrong divisor
    "rope_row_position": ("(t / gw) % gh, t % gw}", "(t / gh) % gw, t % gw}"),
    # large values mapped to the NaN pattern instead of saturating at 448
    "fp8_no_saturation": ("if (a >= 448.0) return (sgn << 7) | 0x7E;", "if (a >= 480.0) return (sgn << 7) | 0x7F;"),
    # e4m3 rounding half away from zero instead of to even
    "fp8_round_half_up": ("double n = nearbyint(a / quantum);", "double n = floor(a / quantum + 0.5);"),
    # padded tokens counted in the block's amax
    "fp8_amax_counts_padding": ("for (int t = t0; t < t0 + blk && t < L; ++t)", "for (int t = t0; t < t0 + blk; ++t)"),
    # e2m1 rounding half away from zero instead of to the even code
    "fp4_round_half_up": ("double r = nearbyint(a / step) * step;", "double r = floor(a / step + 0.5) * step;"),
    # the two elements of a byte swapped between the nibbles
    "fp4_nibble_order": ("codes[((size_t)r * K + c) / 2] = (uint8_t)(lo | (hi << 4));",
                         "codes[((size_t)r * K + c) / 2] = (uint8_t)(hi | (lo << 4));"),
    # scale layout: the row's 32-group and lane swapped inside an atom
    "fp4_sf_layout": ("(size_t)(r % 32) * 16 + (size_t)((r % 128) / 32) * 4", "(size_t)(r % 32) * 4 + (size_t)((r % 128) / 32) * 16"),
    # tensor scale without the e2m1 maximum (448 / amax instead of 6 * 448 / amax)
    "fp4_tensor_scale": ("const float s = amax > 0.0f ? 2688.0f / amax : 1.0f;",
                         "const float s = amax > 0.0f ? 448.0f / amax : 1.0f;"),
    # block scale from the block's amax without dividing by the e2m1 maximum
    "fp4_block_scale": ("float scaled = (bmax / 6.0f) * s;", "float scaled = bmax * s / 448.0f;"),
    # decoded values not divided by the tensor scale
    "fp4_dequant_no_tensor_scale": ("out[(size_t)r * K + c] = oracle_e2m1_decode(code) * scale / (double)s;",
                                    "out[(size_t)r * K + c] = oracle_e2m1_decode(code) * scale;"),
}


# Python-side oracle functions: (function, old text, new text)
PY_MUTANTS = {
    # the receiver takes the sender's heads instead of its own
    "uly_qkv_wrong_heads": ("ulysses_qkv", "x_shards[i][:, :, r * Hg:(r + 1) * Hg, :]",
                            "x_shards[i][:, :, i * Hg:(i + 1) * Hg, :]"),
    # each sender's tokens land in the receiver's own token range
    "uly_qkv_wrong_tokens": ("ulysses_qkv", "dst[:, :, i * Lr:(i + 1) * Lr, :]", "dst[:, :, r * Lr:(r + 1) * Lr, :]"),
    # q, k, v and heads transposed in the attention layout
    "uly_qkv_transposed": ("ulysses_qkv", "deq.transpose(1, 2, 0, 3)", "deq.transpose(2, 1, 0, 3)"),
    # the return exchange puts every sender's heads at the receiver's own head range
    "uly_o_wrong_heads": ("ulysses_o", "dst[:, i * Hg:(i + 1) * Hg, :] = deq", "dst[:, r * Hg:(r + 1) * Hg, :] = deq"),
    # the return exchange takes the sender's token range instead of the receiver's
    "uly_o_wrong_tokens": ("ulysses_o", "o_shards[i][:, r * Lr:(r + 1) * Lr, :]", "o_shards[i][:, i * Lr:(i + 1) * Lr, :]"),
    # the NVFP4 GEMM without its bias, or against B untransposed
    "fp4_gemm_no_bias": ("nvfp4_gemm", "        c = c + np.asarray(bias, dtype=np.float64)[None, :]", "        c = c"),
    "fp4_gemm_bias_per_row": ("nvfp4_gemm", "np.asarray(bias, dtype=np.float64)[None, :]",
                              "np.asarray(bias, dtype=np.float64)[:c.shape[0], None]"),
    # the FP8 attention path with K taken from Q's codes
    "fp8_attention_k_from_q": ("attention_fp8", "kd = dequantize_fp8(k_codes, k_scales, blk)",
                               "kd = dequantize_fp8(q_codes, q_scales, blk)"),
}


def _py_mutant(func_name, old, new):
    src = inspect.getsource(getattr(oracle, func_name))
    assert src.count(old) == 1, f"mutation anchor for {func_name} not unique/present"
    ns = dict(vars(oracle))
    exec(compile(src.replace(old, new), f"<mutant {func_name}>", "exec"), ns)
    return ns[func_name]


def _build_mutant(tmp_path, name, old, new):
    text = open(SRC).read()
    assert text.count(old) == 1, f"mutation anchor for {name} not unique/present"
    path = tmp_path / f"{name}.c"
    path.write_text(text.replace(old, new))
    so = tmp_path / f"{name}.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                           str(path), "-o", str(so), "-lm"])
    return str(so)


def _pin_functions():
    out = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_"):
            continue
        marks = getattr(fn, "pytestmark", [])
        params = [m for m in marks if m.name == "parametrize"]
        if params:
            argname, values = params[0].args[0], params[0].args[1]
            for val in values:
                out.append((f"{name}[{val}]", fn, {argname: val}))
        else:
            out.append((name, fn, {}))
    return out


def _run_pins_with(lib_path):
    saved = oracle._lib
    oracle._lib = None
    real_build = oracle.build
    oracle.build = lambda force=False: lib_path
    failed = []
    try:
        for name, fn, kw in _pin_functions():
            try:
                fn(**kw)
            except Exception:  # AssertionError, or ValueError from a broken selection
                failed.append(name)
    finally:
        oracle.build = real_build
        oracle._lib = saved
    return failed


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(tmp_path, name):
    old, new = MUTANTS[name]
    so = _build_mutant(tmp_path, name, old, new)
    failed = _run_pins_with(so)
    assert failed, f"mutant {name} passed every pin"


@pytest.mark.parametrize("name", sorted(PY_MUTANTS))
def test_pins_catch_python_mutant(monkeypatch, name):
    func_name, old, new = PY_MUTANTS[name]
    monkeypatch.setattr(oracle, func_name, _py_mutant(func_name, old, new))
    failed = _run_pins_with(oracle.build())
    assert failed, f"mutant {name} passed every pin"


def test_real_oracle_passes_all_pins():
    assert _run_pins_with(oracle.build()) == []
    assert ctypes  # keep import
