"""Planted mistakes in the oracle must be caught by its pins (CPU only).

Each mutant is the oracle rebuilt with one known mistake (ORACLE_MUTANT in
engram_oracle.c): a plausible slip in the hash (operator, reset position,
multiplier pairing, remainder sign, sequence reset), in the backward
(accumulation precision, grouping) or in the PLE norm and convolution (scale,
group width, epsilon, dilation, tap order, history reset, residual), in its
backward (SiLU derivative, tap direction, the norm's mean term) or in the
optimizer step (bias correction, epsilon, weight decay). The pins of
test_oracle_hash.py, test_oracle_gather_backward.py, test_oracle_ple.py,
test_oracle_ple_backward.py and test_oracle_adam.py are run against each; at
least one must fail.
"""

import pytest

import oracle
from tests import test_oracle_adam as AD
from tests import test_oracle_gather_backward as GB
from tests import test_oracle_hash as TH
from tests import test_oracle_ple as PL
from tests import test_oracle_ple_backward as PB

HASH_PINS = [
    TH.test_hand_worked_example,
    lambda: [TH.test_bruteforce_adversarial(c, f) for c in range(len(TH.ADVERSARIAL))
             for f in (0, 17)],
    lambda: [TH.test_bruteforce_random(s, 3, 8) for s in range(6)],
    TH.test_single_term_multipliers_isolate_positions,
    TH.test_token_after_eos_hashes_like_sequence_start,
    TH.test_eos_token_keeps_its_own_left_context,
]
BACKWARD_PINS = [
    lambda: [GB.test_backward_matches_add_at(s) for s in range(4)],
    GB.test_backward_bf16_and_f16_decode,
    GB.test_backward_adjoint_identity,
    lambda: GB.test_backward_per_head_mass_and_counts("tiny"),
]

PLE_PINS = [
    lambda: [PL.test_norm_matches_torch_rms_norm(g) for g in (4, 8, 16)],
    PL.test_norm_constant_group_closed_form,
    PL.test_norm_unit_rms_and_branch_scale_invariance,
    PL.test_norm_zero_scale_is_plain_rms_norm,
    lambda: [PL.test_conv_matches_torch_conv1d(K, d, cu) for K, d in ((4, 3), (3, 5))
             for cu in (None, [0, 13, 13, 40])],
    PL.test_conv_impulse_response,
    PL.test_full_tail_matches_torch_chain,
    PL.test_zero_start_convolution_leaves_the_residual,
    PL.test_causal_branch_local_and_sequence_local,
    PL.test_sequences_are_independent,
]

PLE_BWD_PINS = [
    lambda: [PB.test_matches_torch_autograd(*c) for c in PB.CASES],
    lambda: [PB.test_finite_differences(s) for s in range(3)],
    PB.test_linear_convolution_adjoint_and_bilinear_form,
    PB.test_transposed_impulse_response,
    PB.test_norm_input_gradient_orthogonal_to_each_group,
]

ADAM_PINS = [
    AD.test_first_step_closed_form,
    lambda: [AD.test_matches_torch_adamw_when_all_rows_present(wd) for wd in (0.0, 0.05)],
    AD.test_matches_torch_sparse_adam_over_changing_rows,
]

MUTANTS = {
    1: ("add instead of xor", HASH_PINS),
    2: ("reset before EOS instead of after", HASH_PINS),
    3: ("multipliers paired in reverse", HASH_PINS),
    4: ("truncating remainder", HASH_PINS),
    5: ("no reset at cu_seqlens starts", HASH_PINS),
    6: ("fp32 accumulation", BACKWARD_PINS),
    7: ("adjacent rows merged", BACKWARD_PINS),
    8: ("norm scale w instead of 1 + w", PLE_PINS),
    9: ("norm mean over the whole row", PLE_PINS),
    10: ("eps added after the square root", PLE_PINS),
    11: ("dilation off by one", PLE_PINS),
    12: ("conv taps reversed", PLE_PINS),
    13: ("conv history crosses sequence starts", PLE_PINS),
    14: ("residual of the normalised input", PLE_PINS),
    15: ("no bias correction", ADAM_PINS),
    16: ("eps inside the square root", ADAM_PINS),
    17: ("L2 penalty instead of decoupled decay", ADAM_PINS),
    18: ("SiLU derivative taken as the sigmoid", PLE_BWD_PINS),
    19: ("conv gradient sent forward along the taps", PLE_BWD_PINS),
    20: ("norm backward without the mean term", PLE_BWD_PINS),
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_pins_catch_planted_mistake(mutant, tmp_path, monkeypatch):
    what, pins = MUTANTS[mutant]
    monkeypatch.setattr(oracle, "_lib", oracle.build_mutant(mutant, str(tmp_path)))
    caught = []
    for pin in pins:
        try:
            pin()
        except AssertionError:
            caught.append(pin)
    assert caught, f"no pin caught mutant {mutant} ({what})"
