"""The pins catch plausible mistakes in the oracle.

skiparse_oracle.c carries mutation hooks, all off in the normal build: a build with
ORACLE_MUTANT = k plants one plausible mistake -- a wrong group-wise sub-grid position or class,
the 1/sqrt(d) scale dropped, the exponent's sign flipped, padding to a multiple of P instead of
P^2, pad keys left unmasked, the Skiparse-1D frame flattened column-major, the D term dropped
from the backward's dS. Each such build is swapped in for the oracle library and a fixed
selection of the pins is run against it: at least one pin must fail for every mutant, and the
whole selection must pass on the normal build. The builds with a planted mistake stay in
bounds (the oracle skips any slot outside the rearranged tensor), so a mutant can only give
wrong numbers."""

from __future__ import annotations

import pytest

import oracle
import skiparse_synth as synth
import test_oracle_1d_pins as P1
import test_oracle_bwd_pins as PB
import test_oracle_pins as P2
from oracle import build as oracle_build

TOK, GRP = oracle.TOKEN_WISE, oracle.GROUP_WISE
MUTANTS = {1: "group-wise sub-grid position x div P", 2: "group-wise class (x div P^2) mod P",
           3: "softmax scale 1", 4: "exponent sign flipped", 5: "padding to a multiple of P",
           6: "pad keys not masked", 7: "1-D frame flattened column-major",
           8: "backward dS without the D term"}

ANYRES = synth.WORKLOADS["anyres"]
PINS = [
    ("golden class maps", P2.test_class_maps_golden),
    ("golden padding", P2.test_padding_golden),
    ("token-wise = pixel_unshuffle", lambda: P2.test_token_wise_is_pixel_unshuffle(2, 8, 12, 2, 5)),
    ("group-wise = patch unshuffle", lambda: P2.test_group_wise_is_patch_unshuffle(2, 8, 12, 2, 2)),
    ("P = 1 is fp64 SDPA", lambda: P2.test_p1_is_full_attention(2, 5, 6, 2, 16)),
    ("brute force, token-wise", lambda: P2.test_oracle_equals_brute_force(ANYRES, TOK)),
    ("brute force, group-wise", lambda: P2.test_oracle_equals_brute_force(ANYRES, GRP)),
    ("1-D token-wise = strided slicing", lambda: P1.test_token_wise_is_strided_slicing(1, 2, 5, 7, 2)),
    ("1-D group-wise = group reshape", lambda: P1.test_group_wise_is_group_reshape(1, 2, 5, 7, 2)),
    ("1-D brute force", lambda: P1.test_forward_matches_brute_force_mask(TOK, (2, 2, 3, 7, 1, 16), 2)),
    ("backward = autograd", lambda: PB.test_backward_equals_autograd_of_masked_dense_attention(ANYRES, GRP)),
]


def _failures():
    failed = []
    for name, pin in PINS:
        try:
            pin()
        except Exception as e:  # an assertion, or an oracle call the mistake makes fail
            failed.append(f"{name}: {type(e).__name__}")
    return failed


def test_selection_passes_on_the_oracle():
    assert _failures() == []


@pytest.mark.parametrize("k", sorted(MUTANTS), ids=lambda k: f"{k}-{MUTANTS[k].replace(' ', '_')}")
def test_every_planted_mistake_fails_a_pin(k, monkeypatch):
    monkeypatch.setattr(oracle, "_LIB", oracle.load(oracle_build.build(mutant=k)))
    failed = _failures()
    assert failed, f"no pin caught mutant {k} ({MUTANTS[k]})"
