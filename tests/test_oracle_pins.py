"""The CPU oracle against its pins (hand-worked examples, brute force, invariants),
plus a check that every planted mistake in the oracle makes some pin fail."""

import pytest

import oracle
from oracle_pins import ALL_PINS

MUTATIONS = {
    1: "partial block divided by B instead of its key count",
    2: "previous block not forced",
    3: "block ties go to the higher index",
    4: "token causal mask j < i instead of j <= i",
    5: "token ties go to the higher index",
    6: "token score drops the last dimension",
    7: "block scores negated (lowest blocks kept)",
    8: "first block not forced",
    9: "take-all threshold off by one (m+1 blocks kept)",
    10: "attention reads a padding entry as token 0",
    11: "attention scores not scaled",
    12: "attention weights not normalised",
    13: "attention values read from the key rows",
}


@pytest.mark.parametrize("pin", ALL_PINS, ids=[p.__name__ for p in ALL_PINS])
def test_pin(pin):
    assert oracle.get_mutation() == 0
    pin()


@pytest.mark.parametrize("code", sorted(MUTATIONS), ids=[MUTATIONS[c] for c in sorted(MUTATIONS)])
def test_planted_mistake_is_caught(code):
    caught = []
    oracle.set_mutation(code)
    try:
        for pin in ALL_PINS:
            try:
                pin()
            except (AssertionError, oracle.OracleError):
                caught.append(pin.__name__)
    finally:
        oracle.set_mutation(0)
    assert caught, f"no pin caught mutation {code}: {MUTATIONS[code]}"
