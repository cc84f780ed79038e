"""Each plausible mistake planted in a copy of the attention-layer oracle (on
the CPU) must make at least one pin in test_projection_oracle.py fail."""
import importlib.util

import numpy as np
import pytest

import test_projection_oracle as P

MUTANTS = {
    "query_channels_head_minor": ("q = (h @ _f64(w_q).T).reshape(T, HQ, D)",
                                  "q = (h @ _f64(w_q).T).reshape(T, D, HQ).transpose(0, 2, 1)"),
    "key_channels_head_minor": ("k = (h @ _f64(w_k).T).reshape(T, HKV, D)",
                                "k = (h @ _f64(w_k).T).reshape(T, D, HKV).transpose(0, 2, 1)"),
    "value_from_key_weights": ("v = (h @ _f64(w_v).T).reshape(T, HKV, D)",
                               "v = (h @ _f64(w_k).T).reshape(T, HKV, D)"),
    "value_channels_head_minor": ("v = (h @ _f64(w_v).T).reshape(T, HKV, D)",
                                  "v = (h @ _f64(w_v).T).reshape(T, D, HKV).transpose(0, 2, 1)"),
    "output_channel_major": ("y = a.reshape(T, HQ * D) @ _f64(w_o).T",
                             "y = a.transpose(0, 2, 1).reshape(T, HQ * D) @ _f64(w_o).T"),
    "output_weight_reshaped_not_transposed": ("y = a.reshape(T, HQ * D) @ _f64(w_o).T",
                                              "y = a.reshape(T, HQ * D) @ _f64(w_o).reshape(HQ * D, -1)"),
    "rope_dropped": ("pad_mask=pad_mask, window=window, use_rope=use_rope, rope_theta=rope_theta,",
                     "pad_mask=pad_mask, window=window, use_rope=False, rope_theta=rope_theta,"),
}

PINS = [
    P.test_single_token_without_sink_is_value_then_output_projection,
    lambda: P.test_two_tokens_closed_form(False),
    lambda: P.test_two_tokens_closed_form(True),
    lambda: P.test_norm_makes_the_layer_invariant_to_query_and_key_weight_scale("w_q"),
    lambda: P.test_norm_makes_the_layer_invariant_to_query_and_key_weight_scale("w_k"),
    P.test_linear_in_value_and_output_weights,
    P.test_query_heads_within_a_group_are_interchangeable,
    P.test_kv_groups_move_with_their_query_heads,
]


def _load(src, path):
    path.write_text(src.replace("from . import D, HKV, HQ, _f64, attn_fwd",
                                "from oracle import D, HKV, HQ, _f64, attn_fwd"))
    spec = importlib.util.spec_from_file_location("projection_mutant", str(path))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path, monkeypatch):
    import oracle.projection as real
    old, new = MUTANTS[name]
    src = open(real.__file__).read()
    assert src.count(old) == 1, (name, old)
    monkeypatch.setattr(P, "OP", _load(src.replace(old, new), tmp_path / "projection_mutant.py"))
    caught = []
    for pin in PINS:
        try:
            with np.errstate(all="ignore"):
                pin()
        except Exception as e:          # an assertion or a shape failure
            caught.append(type(e).__name__)
    assert caught, "mutant %s passes every pin" % name


def test_unmodified_copy_passes_every_pin(tmp_path, monkeypatch):
    import oracle.projection as real
    monkeypatch.setattr(P, "OP", _load(open(real.__file__).read(), tmp_path / "projection_copy.py"))
    for pin in PINS:
        pin()
