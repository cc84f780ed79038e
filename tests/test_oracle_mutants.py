"""Each plausible mistake planted in a copy of the oracle (on the CPU) must
make at least one of the pins in test_oracle.py fail."""
import os
import subprocess

import numpy as np
import pytest

import oracle
import test_oracle as P

MUTANTS = {
    "rope_sign": ("y[i] = x0 * c - x1 * s;", "y[i] = x0 * c + x1 * s;"),
    "rope_pairing": ("double x0 = x[i], x1 = x[i + HALF];", "double x0 = x[i], x1 = x[(i + 1) % HALF];"),
    "rope_freq": ("pow(theta, -2.0 * (double)i / (double)HD)", "pow(theta, -1.0 * (double)i / (double)HD)"),
    "no_logit_scale": ("double s = dot * scale;", "double s = dot;"),
    "sink_scaled": ("double Z = exp(sink - M);", "double Z = exp(sink * scale - M);"),
    "sink_dropped": ("double Z = exp(sink - M);", "double Z = 0.0 * exp(sink - M);"),
    "window_off_by_one": ("(int64_t)J->window - 1", "(int64_t)J->window"),
    "gqa_modulo": ("const int g = h / (HQ / HKV);", "const int g = h % HKV;"),
    "norm_sum_not_mean": ("sqrt(ss / HD + eps)", "sqrt(ss + eps)"),
    "norm_one_plus_w": ("y[c] = x[c] * r * w[c];", "y[c] = x[c] * r * (1.0 + w[c]);"),
    "causal_off_by_one": [("j <= i; ++j", "j <= (i + 1 < J->T ? i + 1 : i); ++j"),
                          ("if (j > i) return 0;", "if (j > i + 1) return 0;")],
    "doc_mask_dropped": ("if (J->doc[j] < 0 || J->doc[j] != J->doc[i]) return 0;", "if (J->doc[j] < 0) return 0;"),
    "pad_query_lse": ("lse[h] = J->sinks[h];", "lse[h] = 0.0;"),
    "lse_log2": ("lse[h] = M + log(Z);", "lse[h] = M + log2(Z);"),
}

PINS = [
    lambda: P.test_matches_sdpa_with_sink_column(0, False),
    lambda: P.test_matches_sdpa_with_sink_column(7, True),
    P.test_rope_identity_at_zero_and_pair_norms,
    P.test_rope_matches_complex_rotation,
    P.test_rmsnorm_matches_torch,
    P.test_sink_is_unscaled_natural_logit,
    P.test_window_counts_current_token,
    P.test_gqa_head_mapping_is_contiguous_groups,
    P.test_packed_documents_equal_separate_runs,
    P.test_thd_tail_and_padmask_rows_are_padding,
    P.test_hand_computed_four_tokens,
]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    edits = MUTANTS[name]
    if isinstance(edits, tuple):
        edits = [edits]
    src = open(oracle.source_path()).read()
    for old, new in edits:
        assert src.count(old) >= 1, name
        src = src.replace(old, new)
    c = tmp_path / "mutant.c"
    c.write_text(src)
    so = tmp_path / "mutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                           "-D_GNU_SOURCE", str(c), "-o", str(so), "-lm"])
    caught = []
    with oracle.use_library(str(so)):
        for pin in PINS:
            try:
                pin()
            except AssertionError:
                caught.append(pin)
    assert caught, "mutant %s passed every pin" % name
