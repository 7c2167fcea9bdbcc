"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake in a temporary copy of oracle/attn_oracle.c (on the CPU: a dropped term, a wrong
sign, an off-by-one mask, a transposed index), compiles it, swaps it in for the real oracle and checks that at
least one pin of tests/test_oracle_pins.py now fails.
"""
import os
import subprocess

import numpy as np
import pytest

import oracle
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "attn_oracle.c")

MUTATIONS = {
    "dq_drops_scale": ("dQr[j] += scale * dS * K", "dQr[j] += dS * K"),
    "ds_wrong_sign": ("prob[c] * (dP - D)", "prob[c] * (dP + D)"),
    "dk_transposed_row": ("dK[(size_t)c * d + j] += scale * dS * Q[(size_t)r * d + j]",
                          "dK[(size_t)c * d + j] += scale * dS * Q[(size_t)c * d + j]"),
    "dv_drops_prob": ("dV[(size_t)c * d + j] += prob[c] * dOr[j]", "dV[(size_t)c * d + j] += dOr[j]"),
    "causal_off_by_one": ("if (p->causal && c > r)", "if (p->causal && c >= r)"),
    "keylen_off_by_one": ("c >= p->key_lens[b]", "c > p->key_lens[b]"),
    "blockmask_transposed": ("(size_t)(r / p->tile) * nT + (c / p->tile)", "(size_t)(c / p->tile) * nT + (r / p->tile)"),
    "lse_drops_max": ("double lse = m + log(sum);", "double lse = log(sum);"),
    "online_no_l_rescale": ("l[r] *= alpha;", ""),
    "online_no_acc_rescale": ("arow[j] *= alpha;", "arow[j] *= 1.0;"),
    "csr_wrong_index": ("if (mask[(size_t)i * nT + j]) col_idx[nnz++] = j;", "if (mask[(size_t)i * nT + j]) col_idx[nnz++] = i;"),
    "csc_transposed": ("if (mask[(size_t)i * nT + j]) row_idx[nnz++] = i;", "if (mask[(size_t)j * nT + i]) row_idx[nnz++] = i;"),
}

PIN_CALLS = [
    lambda: pins.test_hand_2x2_golden(False),
    lambda: pins.test_hand_2x2_golden(True),
    pins.test_identity_v_exposes_probabilities,
    pins.test_single_rows_match_scipy,
    pins.test_key_length_one_and_causal_first_row,
    lambda: pins.test_online_equals_two_pass(False, 3, 5),
    pins.test_causal_and_key_lens_equal_element_masks,
    pins.test_invisible_tiles_contribute_nothing,
    lambda: pins.test_gradients_match_central_differences(*pins.FD_CASES[0]),
    lambda: pins.test_gradients_match_central_differences(*pins.FD_CASES[3]),
    pins.test_mask_recipe_and_lists_golden,
]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, tmp_path, monkeypatch):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    mutated = tmp_path / "mutant.c"
    mutated.write_text(src.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared", "-o", str(so),
                           str(mutated), "-lm"])
    monkeypatch.setattr(oracle, "_lib", oracle._bind(str(so)))
    failed = []
    for call in PIN_CALLS:
        try:
            with np.errstate(all="ignore"):
                call()
        except AssertionError:
            failed.append(call)
    assert failed, f"no pin caught the planted mistake {name}"
