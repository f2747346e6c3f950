"""Planted-bug checks: each deliberate mistake switched on inside the oracle
(on the CPU) must make at least one pin fail."""
import pytest

import oracle
import oracle_pins

MUTATIONS = {
    1: "bound drops the last channel",
    2: "bound takes min instead of max",
    3: "merge uses the wrong sign in the suffix weight",
    4: "query head h reads KV head h % Hkv (transposed GQA map)",
    5: "ties go to the higher index",
    6: "softmax scale not applied",
    7: "locality uses Qc + Qp instead of Qc - Qp",
    8: "page metadata drops the page's last token",
    9: "union count does not deduplicate",
    10: "log-normaliser misses the running max",
    11: "drift-safe refresh writes the next token's row",
    12: "union variant attends to the row's own pages only",
}


@pytest.mark.parametrize("m", sorted(MUTATIONS), ids=lambda m: MUTATIONS[m])
def test_mutation_is_caught(m):
    caught = []
    oracle.set_mutation(m)
    try:
        for pin in oracle_pins.PINS:
            try:
                pin()
            except AssertionError:
                caught.append(pin.__name__)
    finally:
        oracle.set_mutation(0)
    assert caught, f"mutation {m} ({MUTATIONS[m]}) escaped every pin"
