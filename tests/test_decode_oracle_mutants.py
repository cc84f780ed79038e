"""Each plausible mistake planted in a copy of the decode oracle (on the CPU)
must make at least one of the pins in test_decode_oracle.py fail."""
import importlib.util

import numpy as np
import pytest

import oracle
import test_decode_oracle as P

MUTANTS = {
    "window_off_by_one": ("lo = max(0, p - window + 1) if window > 0 else 0",
                          "lo = max(0, p - window) if window > 0 else 0"),
    "slot_shifted": ("slots = pos % cap", "slots = (pos + 1) % cap"),
    "query_rope_position": ("qt = normalise(q[b, h], q_norm_w, p, use_rope, rope_theta, eps)",
                            "qt = normalise(q[b, h], q_norm_w, p + 1, use_rope, rope_theta, eps)"),
    "key_rope_position": ("k_new[b, g] = normalise(k[b, g], k_norm_w, p, use_rope, rope_theta, eps)",
                          "k_new[b, g] = normalise(k[b, g], k_norm_w, max(p - 1, 0), use_rope, rope_theta, eps)"),
    "sink_dropped": ("z = e.sum() + (np.exp(sink - m) if sink > -np.inf else 0.0)", "z = e.sum()"),
    "sink_scaled": ("z = e.sum() + (np.exp(sink - m) if sink > -np.inf else 0.0)",
                    "z = e.sum() + (np.exp(sink * scale - m) if sink > -np.inf else 0.0)"),
    "gqa_modulo": ("for h in range(GROUP * g, GROUP * (g + 1)):", "for h in range(g, HQ, HKV):"),
    "no_logit_scale": ("s = keys @ qt * scale", "s = keys @ qt"),
    "new_token_excluded": [("keys = np.concatenate([kc[b, g, slots], k_new[b, g][None]], axis=0)",
                            "keys = np.concatenate([kc[b, g, slots], 0.0 * k_new[b, g][None] - 1e30], axis=0)")],
    "lse_log2": ("lse[h, b] = m + np.log(z)", "lse[h, b] = m + np.log2(z)"),
}

PINS = [
    lambda: P.test_decode_equals_last_row_of_prefill(0, 0, False, 4),
    lambda: P.test_decode_equals_last_row_of_prefill(37, 0, True, 64),
    lambda: P.test_decode_equals_last_row_of_prefill(60, 17, True, 17),
    lambda: P.test_decode_equals_last_row_of_prefill(60, 17, True, 23),
    P.test_single_key_closed_form,
    P.test_infinite_sinks,
]


def _load_mutant(src, path):
    spec = importlib.util.spec_from_file_location("decode_mutant", str(path))
    mod = importlib.util.module_from_spec(spec)
    path.write_text(src.replace("from . import D, HKV, HQ, _f64, rmsnorm, rope",
                                "from oracle import D, HKV, HQ, _f64, rmsnorm, rope"))
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path, monkeypatch):
    import oracle.decode as real
    edits = MUTANTS[name]
    if isinstance(edits, tuple):
        edits = [edits]
    src = open(real.__file__).read()
    for old, new in edits:
        assert src.count(old) == 1, (name, old)
        src = src.replace(old, new)
    mutant = _load_mutant(src, tmp_path / "decode_mutant.py")
    monkeypatch.setattr(P, "OD", mutant)
    caught = []
    for pin in PINS:
        try:
            with np.errstate(all="ignore"):
                pin()
        except Exception as e:          # an assertion or a shape/NaN failure
            caught.append(type(e).__name__)
    assert caught, "mutant %s passes every pin" % name


def test_unmodified_copy_passes_every_pin(tmp_path, monkeypatch):
    import oracle.decode as real
    mutant = _load_mutant(open(real.__file__).read(), tmp_path / "decode_copy.py")
    monkeypatch.setattr(P, "OD", mutant)
    for pin in PINS:
        pin()
