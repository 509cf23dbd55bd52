"""Plausible mistakes planted in copies of the oracle must each fail a pin.

Each mutant rewrites one spot of ``oracle/zha_oracle.c`` (a dropped term, a
wrong sign or index, a reversed order, an off-by-one), is compiled into a
temporary library, and the pins of ``pins.py`` are run against it.  The test
passes when at least one pin rejects the mutant -- evidence that the pins
can tell a correct oracle from a broken one.  Everything runs on the CPU.
"""
import os

import pytest

import oracle
from pins import ALL_PINS

SRC = os.path.join(os.path.dirname(oracle.__file__), "zha_oracle.c")

MUTANTS = {
    "leaf_score_without_scale": ("s[i] = scale * dotd(rj, k, d);", "s[i] = dotd(rj, k, d);"),
    "leaf_lse_drops_max": ("m[j] = mx + log(sum);\n        double *gj = g + (size_t)j * d;\n        for (int e = 0;",
                           "m[j] = log(sum);\n        double *gj = g + (size_t)j * d;\n        for (int e = 0;"),
    "parent_lse_drops_max": ("m[j] = mx + log(sum);\n        double *gj = g + (size_t)j * d;\n        for (int k = 0;",
                             "m[j] = log(sum);\n        double *gj = g + (size_t)j * d;\n        for (int k = 0;"),
    "leaf_weights_unnormalised": ("const double w = exp(s[i] - m[j]);", "const double w = exp(s[i] - mx);"),
    "estimate_sign_flipped": ("acc += (q[e] - rj[e]) * gj[e];", "acc += (rj[e] - q[e]) * gj[e];"),
    "estimate_drops_scale": ("const double v = m[j] + scale * acc;", "const double v = m[j] + acc;"),
    "parent_uses_plane0_mass": (
        "e[ch] = orc_estimate(cm + (size_t)ch * R, cg + (size_t)ch * R * d, R, d, ref, rj);",
        "e[ch] = cm[(size_t)ch * R];"),
    "parent_g_wrong_plane": ("const double *cgj = cg + ((size_t)ch * R + j) * d;",
                             "const double *cgj = cg + ((size_t)ch * R) * d;"),
    "plane_offset_sign": ("b[j] = m[j] - scale * dotd(rj, gj, d);\n    }\n    free(k);",
                          "b[j] = m[j] + scale * dotd(rj, gj, d);\n    }\n    free(k);"),
    "topp_tie_order_reversed": ("return (x->id < y->id) ? -1 : (x->id > y->id) ? 1 : 0;",
                                "return (x->id > y->id) ? -1 : (x->id < y->id) ? 1 : 0;"),
    "topp_keeps_one_extra": ("        cum += it[r].p;\n        if (p < 1.0 && cum >= p)\n            done = 1;",
                             "        if (p < 1.0 && cum >= p)\n            done = 1;\n        cum += it[r].p;"),
    "topp_stops_one_early": ("        if (!done) {", "        if (!done && (p >= 1.0 || r == 0 || cum + it[r].p < p)) {"),
    "topp_ignores_p_one": ("if (p < 1.0 && cum >= p)", "if (cum >= p)"),
    "route_children_off_by_one": ("for (int64_t ch = kept[level - 1][k] * c; ch < (kept[level - 1][k] + 1) * c; ++ch)",
                                  "for (int64_t ch = kept[level - 1][k] * c + 1; ch < (kept[level - 1][k] + 1) * c; ++ch)"),
    "sink_dropped": ("if (nleaf == 0 || leaves[0] != 0)\n        tok[T++] = 0;", "if (0)\n        tok[T++] = 0;"),
    "attention_without_scale": ("s[t] = scale * acc;", "s[t] = acc;"),
    "append_skips_ancestors": ("        n /= c;\n    }\n}", "        n /= c;\n        break;\n    }\n}"),
    "node_summary_tail_clip": ("    if (c1 > nbelow)\n        c1 = nbelow;\n    const int nch",
                               "    if (c1 > nbelow)\n        c1 = nbelow - 1;\n    const int nch"),
    "node_summary_leaf_clip": ("            t1 = N;\n        orc_leaf_summary(K, dtype, t0, t1, d, ref, R, m, g, b);",
                               "            t1 = N - 1;\n        orc_leaf_summary(K, dtype, t0, t1, d, ref, R, m, g, b);"),
    "node_summary_child_offset": ("orc_node_summary(K, dtype, N, d, ref, R, c, level - 1, c0 + ch,",
                                  "orc_node_summary(K, dtype, N, d, ref, R, c, level - 1, ch,"),
    "estimate_many_row_offset": ("const int64_t row = level_row0 + ids[i];", "const int64_t row = ids[i];"),
    "decode_heads_ref_stride": ("level_off, R, c, D, ref + (size_t)kh * R * d,", "level_off, R, c, D, ref,"),
    "decode_heads_value_stride": ("const char *Vh = (const char *)V + (size_t)kh * kv_stride * d * esize;",
                                  "const char *Vh = (const char *)V + (size_t)kh * d * esize;"),
    "build_heads_offset_stride": ("b + kh * m_stride, level_off);", "b, level_off);"),
    "growth_when_top_level_is_full": ("if (orc_level_nodes(N, c, D) <= c)", "if (orc_level_nodes(N, c, D) < c)"),
    "grown_level_skips_last_node": ("    for (int64_t n = 0; n < nl; ++n)\n        node_recompute(",
                                    "    for (int64_t n = 0; n + 1 < nl; ++n)\n        node_recompute("),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site of {name} not found exactly once"
    msrc = tmp_path / "mutant.c"
    msrc.write_text(src.replace(old, new))
    lib_path = oracle.compile_oracle(str(msrc), str(tmp_path / "libmutant.so"), openmp=False)
    lib = oracle.load(lib_path)
    caught = []
    for pin in ALL_PINS:
        try:
            pin(lib)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin rejects mutant {name}"
