"""Planted mistakes in the oracle must trip its pins.

Each case compiles a copy of the oracle source with one plausible slip
(dropped scale, wrong kv head, off-by-one visibility, wrong fragment offset,
wrong decoder field, dropped max in lse, flipped merge weight, per-vector
scales dropped, misplaced or misapplied, ...) and runs a
compact subset of the pins against it; at least one must fail.  Mistakes are
planted only in the CPU oracle.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest
import torch

from oracle import oracle as orc
from verify_attention_paged_b200 import workloads as wl
from conftest import to_problem
from test_oracle_pins import sdpa_reference
import test_oracle_append_pins as pins_append
import test_oracle_scale_pins as pins_scale

SRC = os.path.join(os.path.dirname(os.path.dirname(__file__)), "oracle", "lse_oracle.c")

MUTANTS = {
    "scale_dropped": ("x *= pb->scale;", "x *= 1.0;"),
    "wrong_kv_head": ("const int g = h / G;", "const int g = h % pb->n_kv_heads;"),
    "context_off_by_one": ("if (j < C) return 1;", "if (j + 1 < C) return 1;"),
    "mask_bit_shifted": ("(mask >> (j - C)) & 1u", "(mask >> (j - C + 1)) & 1u"),
    "fragment_row_transposed": ("(off * pb->n_kv_heads + g)", "(g * tokens_per_fragment(pb) + off)"),
    "page_index_off": ("int64_t page = j / T;", "int64_t page = (j + 1) / T;"),
    "e4m3_fields": ("decode_minifloat(p[0], 4, 3, 0, 1)", "decode_minifloat(p[0], 5, 2, 0, 1)"),
    "subnormal_exponent": ("pow2(1 - bias - mbits)", "pow2(-bias - mbits)"),
    "lse_drops_max": ("*lse = m + log(l);", "*lse = log(l);"),
    "no_normalisation": ("for (int d = 0; d < D; ++d) out[d] /= l;", ";"),
    "v_through_k_table": ("const uint8_t *v = kv_row(pb, pb->v_pages", "const uint8_t *v = kv_row(pb, pb->k_pages"),
    "merge_weight_sign": ("double w = exp(lp - M);", "double w = exp(M - lp);"),
    "bf16_no_specials": ("8, 7, 1, 0)", "8, 7, 0, 0)"),
    "f16_read_as_bf16": ("5, 10, 1, 0)", "8, 7, 1, 0)"),
    # encoder and K/V append
    "encode_ties_away": ("if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;",
                         "if (frac >= 0.5) r += 1.0;"),
    "encode_subnormal_quantum": ("int be = e - 1 < emin ? emin : e - 1;", "int be = e - 1;"),
    "append_position_off": ("const int64_t pos = (int64_t)seq_lens_before[s] + (i - new_offsets[s]);",
                            "const int64_t pos = (int64_t)seq_lens_before[s] + (i - new_offsets[s]) + 1;"),
    "append_v_through_k_table": ("const int32_t *table = kv ? v_pages : k_pages;",
                                 "const int32_t *table = k_pages;"),
    "e4m3_overflow_not_saturated": ("encode_minifloat(x, 4, 3, 15, 6, 1, 0x7Fu)",
                                    "encode_minifloat(x, 4, 3, 15, 6, 0, 0x7Fu)"),
    # per-vector scales
    "k_scale_dropped": ("(decode_elem(pb->dtype, k + d * es) * sk)",
                        "decode_elem(pb->dtype, k + d * es)"),
    "v_scale_dropped": ("(decode_elem(pb->dtype, v + d * es) * sv)",
                        "decode_elem(pb->dtype, v + d * es)"),
    "scale_block_token_major": ("int64_t at = ((int64_t)frag * pb->n_kv_heads + g) * T + j % T;",
                                "int64_t at = ((int64_t)frag * T + j % T) * pb->n_kv_heads + g;"),
    "v_scale_through_k_table": ("vec_scale(pb, pb->v_pages", "vec_scale(pb, pb->k_pages"),
    "v_scale_in_denominator": ("    l += p;\n", "    l += p * sv;\n"),
    "long_chain_excludes_itself": ("if (!pb->row_masks) return j - C <= r;",
                                   "if (!pb->row_masks) return j - C < r;"),
    "append_not_divided_by_scale": ("const float q = scales ? x[d] / sc : x[d];",
                                    "const float q = x[d];"),
    "append_scale_formats_swapped": ("dtype == ORC_E4M3 ? 448.0f : 57344.0f",
                                     "dtype == ORC_E4M3 ? 57344.0f : 448.0f"),
}


def _build_mutant(tmp_path, name, old, new):
    with open(SRC) as f:
        src = f.read()
    assert src.count(old) >= 1, name
    mutated = src.replace(old, new)
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"{name}.so"
    c.write_text(mutated)
    subprocess.check_call(["gcc", "-std=c99", "-O2", "-fPIC", "-shared", "-o", str(so), str(c),
                           "-lm"])
    return str(so)


def _pins_fail(lib) -> list:
    saved = orc._lib
    failures = []
    orc._lib = None
    try:
        real = orc._load()  # set argtypes on a fresh handle, then swap the library
        m = ctypes.CDLL(lib)
        for fn in ("orc_attention", "orc_attention_one", "orc_attention_split", "orc_decode",
                   "orc_kv_bytes_per_token", "orc_encode", "orc_kv_append"):
            f = getattr(m, fn)
            f.argtypes = getattr(real, fn).argtypes
            f.restype = getattr(real, fn).restype
        orc._lib = m

        def check(name, fn):
            try:
                fn()
            except (AssertionError, orc.OracleError):
                failures.append(name)

        def sdpa(dtype, tree):
            w = wl.small_case(dtype, [37, 20], [3, 4], n_q_heads=4, n_kv_heads=2, head_dim=8,
                              tokens_per_fragment=8, tree=tree, seed=31)
            out, _ = orc.attention(to_problem(w))
            np.testing.assert_allclose(out, sdpa_reference(w), rtol=1e-12, atol=1e-13)

        def split():
            w = wl.small_case("bf16", [37, 20], [3, 4], n_q_heads=4, n_kv_heads=2, head_dim=8,
                              tokens_per_fragment=8, tree=True, seed=32)
            a = orc.attention(to_problem(w))
            b = orc.attention_split(to_problem(w), 7)
            np.testing.assert_allclose(b[0], a[0], rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(b[1], a[1], rtol=1e-12, atol=1e-13)

        def single_key():
            w = wl.small_case("f32", [1], [1], n_q_heads=2, n_kv_heads=1, head_dim=8,
                              tokens_per_fragment=2, seed=33)
            _, lse = orc.attention(to_problem(w))
            k = w.logical_k[0].to(torch.float64).numpy()[0, 0]
            x = w.scale * float(w.q[0, 0].astype(np.float64) @ k)
            assert abs(lse[0, 0] - x) < 1e-12

        def codec(dtype, tdt, nbits):
            codes = np.arange(1 << nbits)
            t = (torch.from_numpy(codes.astype(np.uint8)).view(tdt) if nbits == 8 else
                 torch.from_numpy(codes.astype(np.uint16).view(np.int16)).view(tdt))
            want = t.to(torch.float64).numpy()
            got = np.array([orc.decode(dtype, int(c)) for c in codes])
            assert np.array_equal(np.isnan(want), np.isnan(got))
            assert np.array_equal(want[~np.isnan(want)], got[~np.isnan(got)])

        def encoder(dtype):
            x = pins_append.sample_values(dtype, 3000, seed=12)
            assert np.array_equal(pins_append.encode_all(dtype, x),
                                  pins_append.torch_bits(dtype, x))

        def append(dtype):
            w = wl.small_case(dtype, [40, 9, 1], [1, 2, 1], n_q_heads=4, n_kv_heads=2,
                              head_dim=8, tokens_per_fragment=8, seed=43)
            chunks, st, *_ = pins_append._append_from_logical(w, 11)
            assert st == 0
            for a, b in zip(chunks, w.chunks):
                assert np.array_equal(a, b)

        check("encoder_e4m3", lambda: encoder("e4m3"))
        check("encoder_f16", lambda: encoder("f16"))
        check("encoder_overflow_e4m3", lambda: pins_append.test_overflow_and_nan_rules("e4m3"))
        check("encoder_ties_e5m2", lambda: pins_append.test_encoder_rounds_ties_to_even("e5m2"))
        check("append_bf16", lambda: append("bf16"))
        check("scaled_sdpa_e4m3", lambda: pins_scale.test_scaled_matches_library_sdpa("e4m3", True))
        check("scaled_append_e4m3",
              lambda: pins_append.test_scaled_append_restores_the_generator_bytes_and_scales("e4m3"))
        check("sdpa_bf16_tree", lambda: sdpa("bf16", True))
        check("sdpa_e4m3_chain", lambda: sdpa("e4m3", False))
        check("split", split)
        check("single_key", single_key)
        check("codec_e4m3", lambda: codec("e4m3", torch.float8_e4m3fn, 8))
        check("codec_bf16", lambda: codec("bf16", torch.bfloat16, 16))
        check("codec_f16", lambda: codec("f16", torch.float16, 16))
    finally:
        orc._lib = saved
    return failures


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(tmp_path, name):
    old, new = MUTANTS[name]
    lib = _build_mutant(tmp_path, name, old, new)
    assert _pins_fail(lib), f"mutant {name} passed every pin"


def test_unmutated_source_passes(tmp_path):
    lib = _build_mutant(tmp_path, "identity", "#include <math.h>", "#include <math.h>")
    assert _pins_fail(lib) == []
