"""The CPU oracle against facts fixed by the pages and by mathematics."""
import pytest

from oracle import varq_oracle as O

from oracle_pins import ALL_CHECKS, check_bruteforce_codes


@pytest.mark.parametrize("check", ALL_CHECKS, ids=lambda f: f.__name__)
def test_pin(check):
    check(O)


def test_bruteforce_flags_are_rare():
    # near-tie quotients (where the fp32 definition, not the exact quotient,
    # decides) must stay a small minority of the compared codes
    flagged = check_bruteforce_codes(O, n_cells=700, seed=21)
    assert flagged < 20
