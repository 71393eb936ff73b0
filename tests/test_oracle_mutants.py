"""Plant plausible mistakes in copies of the oracle; each must fail a pin.

The committed oracle is untouched: each mutant is a textual edit of a copy of
paged_oracle.c, compiled into a temporary directory on the CPU.
"""
import os

import pytest

import oracle
from oracle import build as obuild
from oracle_pins import PINS

MUTANTS = {
    "dropped_scale": ("sc[t] = scale * dot;", "sc[t] = dot;"),
    "no_normalisation": ("orow[d] /= Z;", "orow[d] /= 1.0;"),
    "gqa_modulo_grouping": ("const int32_t kvh = h / group;", "const int32_t kvh = h % Hkv;"),
    "no_causal_window": ("const int32_t last = L - q_len + j;", "const int32_t last = L - 1;"),
    "off_by_one_window": ("const int32_t n = last + 1;", "const int32_t n = last;"),
    "pool_layout_transposed": ("return (((size_t)p * (size_t)Hkv + (size_t)kvh) * (size_t)bs + (size_t)o) * (size_t)D;",
                               "return (((size_t)p * (size_t)bs + (size_t)o) * (size_t)Hkv + (size_t)kvh) * (size_t)D;"),
    "half_exponent_bias": ("v = ldexp((double)(frac | 0x400), expo - 25);",
                           "v = ldexp((double)(frac | 0x400), expo - 24);"),
    "subnormal_scale": ("v = ldexp((double)frac, -24);", "v = ldexp((double)frac, -25);"),
    "softmax_sign": ("double w = exp(sc[t] - M);", "double w = exp(M - sc[t]);"),
    "table_index_offset": ("int32_t p = block_tables[(size_t)s * max_blocks_per_seq + t / bs];\n            const uint16_t* vrow",
                           "int32_t p = block_tables[(size_t)s * max_blocks_per_seq + (t + 1) / bs];\n            const uint16_t* vrow"),
    "append_slot_split": ("int32_t o = (int32_t)(slot % bs);\n        for (int32_t h = 0; h < Hkv; ++h) {\n            for (int32_t d = 0; d < D; ++d) {\n                k_pool",
                          "int32_t o = (int32_t)(slot / num_blocks);\n        for (int32_t h = 0; h < Hkv; ++h) {\n            for (int32_t d = 0; d < D; ++d) {\n                k_pool"),
    "q8k_scale_dropped": ("(double)k8[row + d] * (double)k_scales[(size_t)kvh * D + d]", "(double)k8[row + d]"),
    "q8k_scale_ignores_head": ("(double)k_scales[(size_t)kvh * D + d]", "(double)k_scales[(size_t)d]"),
    "q8k_truncating_round": ("rintf(", "truncf("),
    "q8k_scale_over_255": ("(float)amax / 127.0f", "(float)amax / 255.0f"),
    "q8k_append_scale_ignores_head": ("k_code(new_k[src], k_scales[(size_t)h * D + d])", "k_code(new_k[src], k_scales[(size_t)d])"),
    "q8k_no_clamp": ("(r > 127.0f ? 127.0f : r)", "r"),
    "append_k_only": ("v_pool[pool_row(p, h, o, Hkv, bs, D) + d] = new_v[((size_t)t * Hkv + h) * D + d];",
                      "v_pool[pool_row(p, h, o, Hkv, bs, D) + d] = new_k[((size_t)t * Hkv + h) * D + d];"),
    "copy_direction": ("k_pool[dst + e] = k_pool[src + e];", "k_pool[src + e] = k_pool[dst + e];"),
    "formula_missing_factor_2": ("return 2ull * layers", "return 1ull * layers"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(obuild.SRC, encoding="utf-8").read()
    assert src.count(old) == 1, f"mutation site for {name} not unique/found"
    mpath = tmp_path / "mutant.c"
    mpath.write_text(src.replace(old, new), encoding="utf-8")
    so = obuild.build(str(mpath), str(tmp_path / "libmutant.so"), force=True)
    L = oracle.lib(so)
    failed = []
    for pin in PINS:
        try:
            pin(L)
        except Exception as e:  # a pin failing by assertion or by rejecting input
            failed.append(f"{pin.__name__}: {type(e).__name__}")
    assert failed, f"mutant {name} passed every pin"
