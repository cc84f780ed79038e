"""Each plausible mistake planted in a copy of the backward oracle (on the
CPU) must make at least one of the pins in test_backward_oracle.py fail."""
import importlib.util

import numpy as np
import pytest

import test_backward_oracle as P

MUTANTS = {
    "delta_term_dropped": ("dS = P * (dO @ V.T - Dr[:, None])", "dS = P * (dO @ V.T)"),
    "delta_sign": ("dS = P * (dO @ V.T - Dr[:, None])", "dS = P * (dO @ V.T + Dr[:, None])"),
    "dsink_sign": ("dsinks[h] += -np.sum(Psink * Dr)", "dsinks[h] += np.sum(Psink * Dr)"),
    "dsink_without_share": ("dsinks[h] += -np.sum(Psink * Dr)", "dsinks[h] += -np.sum(Dr)"),
    "dv_untransposed": ("dv[a:b, g] += P.T @ dO", "dv[a:b, g] += P @ dO"),
    "dv_one_head_per_group": ("dv[a:b, g] += P.T @ dO",
                              "dv[a:b, g] += (P.T @ dO) if h == GROUP * g else 0.0"),
    "dq_unscaled": ("dqt[a:b, h] = dS @ K * scale", "dqt[a:b, h] = dS @ K"),
    "dk_overwrites_group": ("dkt[a:b, g] += dS.T @ qt[a:b, h] * scale",
                            "dkt[a:b, g] = dS.T @ qt[a:b, h] * scale"),
    "rope_backward_forward_sign": ("dnq = _rope(dqt, pos, rope_theta, -1.0) if use_rope else dqt",
                                   "dnq = _rope(dqt, pos, rope_theta, 1.0) if use_rope else dqt"),
    "key_rope_backward_skipped": ("dnk = _rope(dkt, pos, rope_theta, -1.0) if use_rope else dkt",
                                  "dnk = dkt"),
    "norm_second_term_dropped": ("dx = r * w * dn - x * r ** 3 * t / D", "dx = r * w * dn"),
    "norm_second_term_power": ("dx = r * w * dn - x * r ** 3 * t / D", "dx = r * w * dn - x * r ** 2 * t / D"),
    "norm_weight_grad_without_r": ("dw = np.sum(dn * x * r, axis=(0, 1))", "dw = np.sum(dn * x, axis=(0, 1))"),
    "window_off_by_one": ("allowed &= (i - j) < window", "allowed &= (i - j) <= window"),
    "sink_left_out_of_lse": ("Z = np.exp(S - m[:, None]).sum(axis=1) + np.exp(sink - m)",
                             "Z = np.exp(S - m[:, None]).sum(axis=1)"),
}

PINS = [
    lambda: P.test_gradient_matches_finite_differences("full"),
    lambda: P.test_gradient_matches_finite_differences("sliding_thd"),
    lambda: P.test_gradient_matches_finite_differences("padmask"),
    P.test_padded_tokens_get_zero_gradient,
    P.test_single_token_closed_form,
    P.test_value_gradient_column_sum,
    P.test_norm_scale_invariance_makes_gradient_orthogonal,
    P.test_packed_documents_equal_separate_runs,
    P.test_infinite_sinks,
    P.test_default_positions_are_document_local,
]


def _load_mutant(src, path):
    path.write_text(src.replace("from . import D, HKV, HQ, _f64, doc_ids",
                                "from oracle import D, HKV, HQ, _f64, doc_ids"))
    spec = importlib.util.spec_from_file_location("backward_mutant", str(path))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path, monkeypatch):
    import oracle.backward as real
    old, new = MUTANTS[name]
    src = open(real.__file__).read()
    assert src.count(old) == 1, (name, old)
    mutant = _load_mutant(src.replace(old, new), tmp_path / "backward_mutant.py")
    monkeypatch.setattr(P, "OB", mutant)
    caught = []
    for pin in PINS:
        try:
            with np.errstate(all="ignore"):
                pin()
        except Exception as e:          # an assertion or a shape/NaN failure
            caught.append(type(e).__name__)
    assert caught, "mutant %s passes every pin" % name


def test_unmodified_copy_passes_every_pin(tmp_path, monkeypatch):
    import oracle.backward as real
    mutant = _load_mutant(open(real.__file__).read(), tmp_path / "backward_copy.py")
    monkeypatch.setattr(P, "OB", mutant)
    for pin in PINS:
        pin()
