"""The tensor-core decode kernel's ring protocol, checked on the CPU: the model
in tests/ring_protocol_model.py must hold under random interleavings, and
with any one of its rules switched off the checks must fail."""

import pytest

from tests.ring_protocol_model import RULES, run_schedules


def test_protocol_holds_over_random_schedules():
    run_schedules(1500, seed=7)


@pytest.mark.parametrize("rule", RULES)
def test_a_broken_rule_is_caught(rule):
    with pytest.raises(AssertionError):
        run_schedules(3000, seed=11, rules=tuple(r for r in RULES if r != rule))
