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


def test_harness_tables_follow_the_schedule():
    # the next-frame workloads' input tables (4,680-token chunks of three
    # 1,560-token frames) are the oracle's schedule with frames counted over
    # the whole cache
    import numpy as np
    from packed_kv_attention_b200 import synth
    T = 4680 * 3 + 777
    c1, s1 = synth.rope_tables_3d(T, 128)
    c2, s2 = O.rope_schedule_tables(T, 1560, 52, synth.rope_axis_pairs(128))
    assert np.array_equal(c1.numpy(), c2) and np.array_equal(s1.numpy(), s2)
