"""The oracle pins have teeth: each plausible mistake, planted in a copy of the
oracle's C source and compiled on the CPU, must make at least one pin fail
(pins of tests/test_oracle.py, test_oracle_rope.py, test_oracle_fp8.py and test_oracle_prefill.py).

The mutant library replaces the oracle's loaded library only for the duration
of one test; the real oracle source is never modified.
"""
import inspect
import os
import subprocess
import tempfile

import pytest

import oracle
from tests import test_oracle as pins
from tests import test_oracle_fp8 as fp8_pins
from tests import test_oracle_prefill as prefill_pins
from tests import test_oracle_rope as rope_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "pa_oracle.c")

MUTANTS = {
    # query head h reads kv head h % Hkv instead of h / (Hq/Hkv)
    "gqa_modulo_grouping": ("return h / (num_q_heads / num_kv_heads);",
                            "return h % num_kv_heads;"),
    # the softmax scale is dropped
    "scale_dropped": ("s[j - t0] = scale * dot;", "s[j - t0] = dot;"),
    # offset inside a block off by one
    "offset_off_by_one": ("const int64_t offset = position % block_size;",
                          "const int64_t offset = (position + 1) % block_size;"),
    # pool read as [N][Bs][Hkv][D] (head and offset axes transposed)
    "pool_axes_transposed": (
        "return ((block * num_kv_heads + kv_head) * block_size + offset) * head_dim + d;",
        "return ((block * block_size + offset) * num_kv_heads + kv_head) * head_dim + d;"),
    # weights not normalised
    "softmax_not_normalised": ("const double p = exp(s[j - t0] - m) / Z;",
                               "const double p = exp(s[j - t0] - m);"),
    # the newest token is left out of the context
    "last_token_dropped": ("for (int64_t j = t0; j < t1; ++j) {\n        double dot",
                           "for (int64_t j = t0; j + 1 < t1; ++j) {\n        double dot"),
    # log-sum-exp loses the running max
    "lse_without_max": ("return m + log(Z);", "return log(Z);"),
    # merge weights with the wrong sign in the exponent
    "merge_weight_sign": ("const double w = exp(lse[s] - M);", "const double w = exp(M - lse[s]);"),
    # append writes V's row into the K cache
    "append_k_from_v": ("k_cache[dst] = k[src];", "k_cache[dst] = v[src];"),
    # append ignores the skip marker and writes a slot -1 token to slot 0
    "append_negative_not_skipped": ("const int64_t slot = slot_mapping[t];",
                                    "const int64_t slot = slot_mapping[t] < 0 ? 0 : slot_mapping[t];"),
    # K and V swapped in the gather
    "k_v_swapped": ("gather_sequence(k_cache, table_row, L, kvh", "gather_sequence(v_cache, table_row, L, kvh"),
    # RoPE: rotation sense flipped
    "rope_sign": ("yr[i] = x1 * c - x2 * s;", "yr[i] = x1 * c + x2 * s;"),
    # RoPE: frequency exponent i/D instead of 2i/D
    "rope_exponent": ("pow(theta, -2.0 * (double)i / (double)D)", "pow(theta, -1.0 * (double)i / (double)D)"),
    # RoPE: wrong partner (neighbour instead of the other half)
    "rope_pairing": ("const double x2 = oracle_bf16_to_double(xr[i + half]);",
                     "const double x2 = oracle_bf16_to_double(xr[(i + 1) % D]);"),
    # RoPE: position off by one
    "rope_position": ("const double a = (double)pos[t] *", "const double a = (double)(pos[t] + 1) *"),
    # bf16 rounding truncates instead of rounding to nearest
    "round_truncates": ("v = ldexp(rint(ldexp(v, -qexp)), qexp);", "v = ldexp(trunc(ldexp(v, -qexp)), qexp);"),
    # E4M3: exponent bias off by one
    "e4m3_bias": ("v = ldexp(1.0 + (double)m / 8.0, e - 7);", "v = ldexp(1.0 + (double)m / 8.0, e - 6);"),
    # E4M3: subnormal step 2^-10 instead of 2^-9
    "e4m3_subnormal": ("v = ldexp((double)m, -9);", "v = ldexp((double)m, -10);"),
    # E4M3: no saturation below the next binade
    "e4m3_saturation": ("if (a >= 448.0) return sign | 0x7E;", "if (a >= 480.0) return sign | 0x7E;"),
    # E4M3: ties away from zero
    "e4m3_ties_away": ("a = ldexp(rint(ldexp(a, -qexp)), qexp);", "a = ldexp(round(ldexp(a, -qexp)), qexp);"),
    # E4M3 quantization divides by the inverse scale
    "e4m3_quantize_scale": ("volatile float y = f * inv_scale;", "volatile float y = f / inv_scale;"),
    # FP8 decode: V scale dropped; K and V scales swapped
    "e4m3_decode_v_scale": ("gather_sequence_e4m3(v_cache, v_scale,", "gather_sequence_e4m3(v_cache, 1.0,"),
    "e4m3_decode_scales_swapped": ("gather_sequence_e4m3(k_cache, k_scale,", "gather_sequence_e4m3(k_cache, v_scale,"),
    # prefill: causal limit off by one, query positions from 0, query rows not offset
    "prefill_causal": ("attend(qd, K, V, 0, pos + 1, head_dim", "attend(qd, K, V, 0, pos, head_dim"),
    "prefill_position": ("const int64_t pos = L - Tq + i;", "const int64_t pos = i;"),
    "prefill_rows": ("const int64_t row = (q0 + i) * num_q_heads + h;", "const int64_t row = i * num_q_heads + h;"),
    # bf16 rounding breaks ties away from zero instead of to even
    "round_ties_away": ("v = ldexp(rint(ldexp(v, -qexp)), qexp);", "v = ldexp(round(ldexp(v, -qexp)), qexp);"),
}


def _pin_calls():
    """Every pin in test_oracle as a zero-argument callable (parametrised ones expanded)."""
    calls = []
    members = (inspect.getmembers(pins, inspect.isfunction) + inspect.getmembers(rope_pins, inspect.isfunction)
               + inspect.getmembers(fp8_pins, inspect.isfunction)
               + inspect.getmembers(prefill_pins, inspect.isfunction))
    for name, fn in members:
        if not name.startswith("test_"):
            continue
        marks = getattr(fn, "pytestmark", [])
        params = [m for m in marks if m.name == "parametrize"]
        if not params:
            calls.append((name, fn, {}))
            continue
        mark = params[0]
        argnames = [a.strip() for a in mark.args[0].split(",")] if isinstance(mark.args[0], str) else list(mark.args[0])
        for values in mark.args[1]:
            values = values if len(argnames) > 1 else (values,)
            calls.append((name, fn, dict(zip(argnames, values))))
    return calls


def _build_mutant(old, new, tmpdir):
    src = open(SRC).read()
    assert src.count(old) >= 1, "mutation anchor not found: %r" % old
    src = src.replace(old, new, 1)
    path_c = os.path.join(tmpdir, "mutant.c")
    path_so = os.path.join(tmpdir, "mutant.so")
    open(path_c, "w").write(src)
    subprocess.check_call(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c11", path_c,
                           "-o", path_so, "-lm"])
    return path_so


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_pins_catch_planted_mistake(mutant, monkeypatch):
    import ctypes
    old, new = MUTANTS[mutant]
    real = oracle._lib()
    with tempfile.TemporaryDirectory() as tmp:
        so = _build_mutant(old, new, tmp)
        mut = ctypes.CDLL(so)
        # reuse the real library's prototypes on the mutant's symbols
        for sym in ("oracle_bf16_to_double", "oracle_kv_bytes", "oracle_slot", "oracle_slot_mapping",
                    "oracle_append_kv", "oracle_paged_decode", "oracle_paged_decode_partial",
                    "oracle_merge_partials", "oracle_set_num_threads", "oracle_num_threads",
                    "oracle_rope", "oracle_round_bf16", "oracle_e4m3_to_double", "oracle_e4m3_from_float",
                    "oracle_quantize_e4m3", "oracle_append_kv_e4m3", "oracle_paged_decode_e4m3",
                    "oracle_paged_prefill"):
            f_real, f_mut = getattr(real, sym), getattr(mut, sym)
            f_mut.argtypes = f_real.argtypes
            f_mut.restype = f_real.restype
        monkeypatch.setattr(oracle, "_LIB", mut)
        caught = []
        for name, fn, kwargs in _pin_calls():
            try:
                fn(**kwargs)
            except AssertionError:
                caught.append(name)
        assert caught, "no pin caught mutant %s" % mutant
