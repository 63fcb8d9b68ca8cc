"""Planted mistakes: a mutated copy of the oracle must fail the pins (CPU only).

Each case edits one plausible mistake into a copy of oracle.c (a wrong group
index, an off-by-one causal bound, a dropped scale or RoPE term, a transposed
weight, the wrong up-projection, a missing log, another head's values, a
missing normalisation of the merge or of the probabilities, a cache expansion
that copies the wrong RoPE key or uses the key weight for the value), compiles
it into a temporary library and runs one of
the pins of test_oracle_pins.py against it: the pin must fail.  This shows the
pins can tell the definition from its likely corruptions.
"""
import os
import subprocess

import pytest

import oracle
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

MUTATIONS = {
    "group_index_modulo": (
        "int group = i / (c->h_q / c->h_kv); /* repeat_interleave grouping */",
        "int group = i % c->h_kv;",
        lambda: pins.test_gqa_matches_library_sdpa(8, 2, False, 2)),
    "causal_off_by_one": (
        "return causal ? L - s_q + t + 1 : L;",
        "return causal ? L - s_q + t : L;",
        lambda: pins.test_bottom_right_reading_differs_from_top_left()),
    "scale_dropped": (
        "            s[j] = c->scale * acc;\n        }\n        softmax_combine(s, n, V, c->d, c->d,",
        "            s[j] = acc;\n        }\n        softmax_combine(s, n, V, c->d, c->d,",
        lambda: pins.test_gqa_matches_library_sdpa(8, 8, True, 1)),
    "rope_term_dropped": (
        "                for (int e = 0; e < c->d_r; ++e) acc += qr[e] * kr[e];\n",
        "",
        lambda: pins.test_latent_expanded_matches_library(True)),
    "weight_transposed": (
        "                ak += Wk[(long)e * c->r_kv + r] * cj[r];",
        "                ak += Wk[(long)r * c->d_h + e] * cj[r];",
        lambda: pins.test_latent_expanded_matches_library(False)),
    "absorbed_wrong_up_projection": (
        "            for (int r = 0; r < c->r_kv; ++r) a += Wv[(long)e * c->r_kv + r] * ot[r];",
        "            for (int r = 0; r < c->r_kv; ++r) a += Wk[(long)e * c->r_kv + r] * ot[r];",
        lambda: pins.test_absorbed_equals_expanded(1)),
    "lse_without_log": (
        "    if (lse) *lse = m + log(z);",
        "    if (lse) *lse = m + z;",
        lambda: pins.test_zero_scale_is_prefix_mean()),
    "gta_group_values": (
        "const double *V = c->v + ((long)b * c->H + h) * c->Lmax * c->d_v;",
        "const double *V = c->v + ((long)b * c->H + gamma * per_group) * c->Lmax * c->d_v;",
        lambda: pins.test_gta_matches_library(3, 12, True)),
    "merge_unnormalised": (
        "        out[d] = a / z;",
        "        out[d] = a;",
        lambda: pins.test_merge_of_disjoint_partials_equals_full_attention()),
    "probs_unnormalised": (
        "    for (int j = 0; j < n; ++j) p[j] = exp(p[j] - m) / z;",
        "    for (int j = 0; j < n; ++j) p[j] = exp(p[j] - m);",
        lambda: pins.test_probabilities_sum_to_one_and_reproduce_output()),
    "expand_cache_rope_from_latent": (
        "c->kr[((long)b * c->Lmax + j) * c->d_r + e] = cj[c->r_kv + e];",
        "c->kr[((long)b * c->Lmax + j) * c->d_r + e] = cj[e];",
        lambda: pins.test_expand_cache_then_gqa_equals_latent()),
    "expand_cache_value_weight": (
        "                av += Wv[(long)e * c->r_kv + r] * cj[r];\n            }\n            ko[e] = ak;",
        "                av += Wk[(long)e * c->r_kv + r] * cj[r];\n            }\n            ko[e] = ak;",
        lambda: pins.test_expand_cache_then_gqa_equals_latent()),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, tmp_path, monkeypatch):
    old, new, pin = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    mutated = tmp_path / "oracle_mutant.c"
    mutated.write_text(src.replace(old, new, 1))  # first site only
    so = tmp_path / "liboracle_mutant.so"
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-pthread", "-o", str(so), str(mutated), "-lm"],
                   check=True)
    monkeypatch.setattr(oracle, "_lib", oracle.load_library(str(so)))
    with pytest.raises(AssertionError):
        pin()
    # the unmutated oracle passes the same pin
    monkeypatch.setattr(oracle, "_lib", None)
    pin()
