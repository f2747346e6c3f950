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
    13: "row-by-row dense pass decodes the head modulo Hkv instead of Hq",
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


# Planted mistakes in the variable-length reading (the Python layer that lays
# one-sequence problems side by side): each must make a varlen pin fail.
def _varlen_pins():
    return [p for p in oracle_pins.PINS if p.__name__.startswith("pin_varlen")]


def _wrong_prefix(X, s, L):  # one token past the sequence's end
    return oracle.f32(X[s:s + 1, :, :int(L) + 1])


def _wrong_seq(X, s, L):  # the next sequence's tokens
    t = (s + 1) % X.shape[0]
    return oracle.f32(X[t:t + 1, :, :int(L)])


def _wrong_shape(sh, L):  # each sequence one token short (never past its slice)
    return oracle.shape(1, sh.Hq, sh.Hkv, sh.d, max(1, int(L) - 1), sh.ps, sh.B, sh.A,
                        sh.budget, sh.scale, sh.flags)


VARLEN_MUTATIONS = {
    "reads one token past each sequence": ("_seq_prefix", _wrong_prefix),
    "reads the next sequence's prefix": ("_seq_prefix", _wrong_seq),
    "drops each sequence's last token": ("seq_shape", _wrong_shape),
}


@pytest.mark.parametrize("name", sorted(VARLEN_MUTATIONS))
def test_varlen_mutation_is_caught(name, monkeypatch):
    attr, fn = VARLEN_MUTATIONS[name]
    monkeypatch.setattr(oracle, attr, fn)
    caught = []
    for pin in _varlen_pins():
        try:
            pin()
        except (AssertionError, ValueError, IndexError):
            caught.append(pin.__name__)
    assert caught, f"varlen mutation '{name}' escaped every pin"
