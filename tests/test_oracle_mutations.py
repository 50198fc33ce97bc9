"""Mutation check of the oracle pins: plant one plausible mistake at a time in
a copy of oracle.c (on the CPU, in a temporary directory), rebuild it, and
assert that at least one pin fails.  A pin set that let a planted mistake
through would not be pinning the oracle."""
import os
import subprocess

import numpy as np
import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

MUTATIONS = {
    "alibi_sign": ("val += -slopes[h] * fabs((double)(i - j));",
                   "val += slopes[h] * fabs((double)(i - j));"),
    "causal_strict": ("if (m->causal && j > i) return 0;",
                      "if (m->causal && j >= i) return 0;"),
    "padding_off_by_one": ("if (m->kv_len && j >= m->kv_len[b]) return 0;",
                           "if (m->kv_len && j > m->kv_len[b]) return 0;"),
    "lse_without_max": ("lse[i] = mx + log(sum);", "lse[i] = log(sum);"),
    "dk_without_scale": ("dkh[(int64_t)j * D + d] = scale * acc;",
                         "dkh[(int64_t)j * D + d] = acc;"),
    "ds_sign": ("ds[(int64_t)i * Sk + j] = pij * (ds[(int64_t)i * Sk + j] - dl);",
                "ds[(int64_t)i * Sk + j] = pij * (dl - ds[(int64_t)i * Sk + j]);"),
    "modality_transposed": ("else if (a == 0 && c == 1) ok = m->allow01;",
                            "else if (a == 0 && c == 1) ok = m->allow10;"),
    "diagonal_ignored": ("if (m->allow_diag && i == j) ok = 1;",
                         "if (m->allow_diag && i == j) ok = ok;"),
    "diagonal_on_ids": ("if (m->allow_diag && i == j) ok = 1;",
                        "if (m->allow_diag && a == c) ok = 1;"),
    "additive_ignored": ("if (m && m->add) val += m->add[b * m->asb + h * m->ash + (int64_t)i * m->asq + j];",
                         "if (m && m->add) val += 0.0;"),
    "additive_transposed": ("if (m && m->add) val += m->add[b * m->asb + h * m->ash + (int64_t)i * m->asq + j];",
                            "if (m && m->add) val += m->add[b * m->asb + h * m->ash + (int64_t)(j % Sq) * m->asq + (i % Sk)];"),
    "additive_sign": ("if (m && m->add) val += m->add[b * m->asb + h * m->ash + (int64_t)i * m->asq + j];",
                      "if (m && m->add) val -= m->add[b * m->asb + h * m->ash + (int64_t)i * m->asq + j];"),
    "additive_neginf_kept": ("      if (val == -INFINITY) { /* an additive -inf masks the pair */",
                             "      if (0) { /* an additive -inf masks the pair */"),
    "philox_round_order": ("    x0 = hi1 ^ x1 ^ k0;", "    x0 = hi0 ^ x1 ^ k0;"),
    "dropout_counter_transposed": ("  uint32_t ctr[4] = {(uint32_t)block, (uint32_t)(block >> 32), (uint32_t)i, (uint32_t)bh};",
                                   "  uint32_t ctr[4] = {(uint32_t)block, (uint32_t)(block >> 32), (uint32_t)bh, (uint32_t)i};"),
    "dropout_block_of_16_keys": ("  uint64_t block = m->offset + (uint64_t)(j / 8);",
                                 "  uint64_t block = m->offset + (uint64_t)(j / 16);"),
    "dropout_key_halves_swapped": ("  uint32_t key[2] = {(uint32_t)m->seed, (uint32_t)(m->seed >> 32)};",
                                   "  uint32_t key[2] = {(uint32_t)(m->seed >> 32), (uint32_t)m->seed};"),
    "dropout_field_order": ("  uint32_t u = (w[f / 2] >> (16 * (f % 2))) & 0xFFFFu;",
                            "  uint32_t u = (w[f % 4] >> (16 * (f / 4))) & 0xFFFFu;"),
    "philox_weyl_constant": ("  const uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;",
                             "  const uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE87u;"),
    "dropout_no_rescale": ("(dropout_keep(m, N, b, h, i, j) ? 1.0 / m->keep_prob : 0.0)",
                           "(dropout_keep(m, N, b, h, i, j) ? 1.0 : 0.0)"),
    "dropout_dp_unmasked": ("        dp *= f[(int64_t)i * Sk + j];", "        dp *= 1.0;"),
    "dq_uses_q": ("acc += ds[(int64_t)i * Sk + j] * kh[(int64_t)j * D + d];",
                  "acc += ds[(int64_t)i * Sk + j] * qh[(int64_t)j * D + d];"),
}

CHECKS = [
    lambda: pins.test_hand_two_keys("none"),
    lambda: pins.test_hand_two_keys("causal"),
    pins.test_alibi_q0_closed_form,
    lambda: pins.test_q_zero_gives_mean_of_allowed_v("padding"),
    lambda: pins.test_q_zero_gives_mean_of_allowed_v("modality"),
    lambda: pins.test_hand_cross_modal_diagonal("page_rule"),
    lambda: pins.test_hand_cross_modal_diagonal("image_only_with_diag"),
    lambda: pins.test_matches_torch_sdpa_fwd_bwd("causal", (13, 13)),
    lambda: pins.test_matches_torch_sdpa_fwd_bwd("padding", (7, 19)),
    lambda: pins.test_bwd_finite_differences("none", True),
    lambda: pins.test_bias_of_zero_and_neginf_equals_the_bool_mask("bool"),
    lambda: pins.test_bias_constant_shift_moves_only_the_lse((2, 3, 6, 9)),
    pins.test_bias_q0_closed_form,
    pins.test_philox_known_answer_vectors,
    pins.test_philox_matches_torch_engine,
    lambda: pins.test_dropout_mask_layout_matches_torch_philox(77),
    lambda: pins.test_dropout_matches_torch_autograd("causal"),
]


def _any_check_fails():
    for chk in CHECKS:
        try:
            chk()
        except (AssertionError, RuntimeError):
            return True
    return False


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, tmp_path):
    before, after = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(before) == 1, f"mutation anchor for {name} not found once"
    mutated = tmp_path / "oracle_mut.c"
    mutated.write_text(src.replace(before, after))
    so = tmp_path / "liboracle_mut.so"
    subprocess.run(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-std=c11",
                    "-o", str(so), str(mutated), "-lm"], check=True)
    with oracle.use_library(str(so)):
        assert _any_check_fails(), f"planted mistake '{name}' passed every pin"


def test_unmutated_oracle_passes_the_same_checks():
    assert not _any_check_fails()
