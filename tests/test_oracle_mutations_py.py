"""Planted mistakes in the Python half of the oracle: a mutated copy must fail the pins (CPU only).

The paged, top-k sparse and FP8 parts of the oracle are plain Python in ``oracle/__init__.py`` (the page-table
lookup, the choice of the keys a sparse query counts, the e4m3 decode and its per-head scale).  Each case here
edits one plausible mistake into a copy of that source, loads the copy as a separate module and runs one pin of
test_oracle_pins.py against it: the pin must fail, and the unmutated oracle passes the same pin.
"""
import os
import types

import pytest

import oracle
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "__init__.py")

MUTATIONS = {
    # the e4m3 exponent bias taken as 8 instead of 7
    "e4m3_exponent_bias": ("np.exp2(e - 7.0)", "np.exp2(e - 8.0)", pins.test_e4m3_decoding_and_fp8_oracle),
    # subnormals scaled as m * 2^-10 instead of m * 2^-9
    "e4m3_subnormal_scale": ("m * 2.0 ** -9", "m * 2.0 ** -10", pins.test_e4m3_decoding_and_fp8_oracle),
    # the per-KV-head dequantisation scale forgotten
    "fp8_scale_dropped": ("return decode_e4m3(x) * _f64(head_scale)[None, :, None, None]", "return decode_e4m3(x)",
                          pins.test_e4m3_decoding_and_fp8_oracle),
    # the block table ignored: pages read as if the pool were in sequence order
    "page_table_ignored": ("out[b, :, t0:t0 + n, :] = pages[bt[b, j], :, :n, :]",
                           "out[b, :, t0:t0 + n, :] = pages[(b * bt.shape[1] + j) % num_pages, :, :n, :]",
                           pins.test_paged_oracle_shuffled_pool_and_shared_prefix),
    # the query token's own key left out of its sparse selection (strict causal bound)
    "sparse_causal_bound": ("if 0 <= j <= last]", "if 0 <= j < last]",
                            pins.test_sparse_oracle_full_selection_equals_dense_causal),
    # the per-group sparse path with the shared RoPE key's term dropped from the scores
    "expanded_sparse_rope_dropped": ("o, l = gqa(np.concatenate([qs[0], qs[1]], -1), key, val, lens, False, scale)",
                                     "o, l = gqa(np.concatenate([qs[0], 0 * qs[1]], -1), key, val, lens, False, scale)",
                                     pins.test_expanded_sparse_full_selection_equals_latent_definition),
    # the per-group sparse path attending to the expanded keys as values
    "expanded_sparse_value_is_key": ("val = np.concatenate([cs[1], np.zeros(", "val = np.concatenate([cs[0], np.zeros(",
                                     pins.test_expanded_sparse_full_selection_equals_latent_definition),
    # padding entries (-1) not skipped: they index the last cache row
    "sparse_padding_kept": ("if 0 <= j <= last]", "if j <= last]",
                            pins.test_sparse_oracle_subset_equals_dense_over_the_subset_and_skips_junk),
}


def _mutant(old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site not found once: {old!r}"
    mod = types.ModuleType("oracle_mutant")
    mod.__file__ = SRC
    exec(compile(src.replace(old, new), SRC, "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake_in_python_oracle(name, monkeypatch):
    old, new, pin = MUTATIONS[name]
    monkeypatch.setattr(pins, "oracle", _mutant(old, new))
    with pytest.raises(AssertionError):
        pin()
    monkeypatch.setattr(pins, "oracle", oracle)
    pin()
