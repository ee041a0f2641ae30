"""The Python oracle against facts the pages and mathematics fix (CPU only)."""

import pins


def test_golden_page_examples():
    """Values printed by the pages (tests/golden/page_examples.txt)."""
    assert pins.golden_failures() == []


def test_target_test_probes():
    """Closed-form outcomes of the five target tests (internal precision,
    rounding mode, normalisation stage, subnormal behaviour, write-back) and
    the special-value readings."""
    assert pins.probe_failures() == []


def test_neutral_subgroups_algorithm4():
    """Obs. 2 / Algorithm 4: Ampere's only nontrivial neutral subgroup is
    {C, P[1..8]}; Hopper has none."""
    assert pins.neutral_failures() == []


def test_bf16_threshold_and_minimum_contribution():
    """Recovered pipeline, BF16 paragraph: smallest contribution 2^-156 and
    the max-exponent threshold -133."""
    assert pins.floor_failures() == []


def test_tile_indexing():
    assert pins.tile_failures() == []


def test_random_elements_match_rational_restatement():
    assert pins.rational_failures(n_per_pair=150, seed=2024) == []
