"""The step kernel's exact rescoring of a page bound picks one operand per
channel (kmax where q >= 0, i.e. its sign bit is clear; kmin elsewhere)
instead of taking max(q*kmax, q*kmin) as the QUEST bound is written (LoSA
paper, methodology: QUEST page selection; QUEST paper, criticality
estimation).  This checks, on the CPU in float32, that the channel-order sum
with that choice is bit for bit the sum with the max for bf16 operands with
kmin <= kmax: random pages, and pages built from the hard values (signed
zeros, bf16 subnormals, values whose products overflow).  The GPU parity
tests check the kernel itself against the oracle."""
import numpy as np


def _bf16(x):
    """Round-toward-zero bf16 values as float32 (any bf16 bit pattern)."""
    b = np.asarray(x, dtype=np.float32).view(np.uint32) & np.uint32(0xFFFF0000)
    return b.view(np.float32)


def _sums(q, kmin, kmax):
    """(max form, operand-choice form) channel-order float32 sums per page;
    q [d], kmin/kmax [P, d]."""
    acc_max = np.zeros(kmin.shape[0], dtype=np.float32)
    acc_sel = np.zeros(kmin.shape[0], dtype=np.float32)
    with np.errstate(over="ignore", invalid="ignore"):
        for i in range(q.shape[0]):
            a = q[i] * kmax[:, i]
            b = q[i] * kmin[:, i]
            acc_max = acc_max + np.fmax(a, b)
            k = kmin[:, i] if np.signbit(q[i]) else kmax[:, i]
            acc_sel = acc_sel + q[i] * k
    return acc_max, acc_sel


def _same(x, y):
    """Equal values (-0 == +0), or both NaN."""
    return np.all((x == y) | (np.isnan(x) & np.isnan(y)))


def _pages(rng, P, d, pool=None):
    if pool is None:
        a = _bf16(rng.standard_normal((P, d)).astype(np.float32))
        b = _bf16(rng.standard_normal((P, d)).astype(np.float32))
    else:
        a = _bf16(rng.choice(pool, size=(P, d)))
        b = _bf16(rng.choice(pool, size=(P, d)))
    return np.minimum(a, b), np.maximum(a, b)


def test_operand_choice_matches_max_random():
    rng = np.random.default_rng(7)
    d = 128
    for _ in range(20):
        q = _bf16(rng.standard_normal(d).astype(np.float32) * rng.choice([1e-3, 1.0, 30.0]))
        kmin, kmax = _pages(rng, 256, d)
        m, s = _sums(q, kmin, kmax)
        assert _same(m, s)


def test_operand_choice_matches_max_hard_values():
    rng = np.random.default_rng(11)
    d = 64
    sub = np.float32(np.uint32(0x00010000).view(np.float32))  # a bf16 subnormal
    pool = np.array([0.0, -0.0, sub, -sub, 1.0, -1.0, 2.0 ** -120, -(2.0 ** -120), 3e38, -3e38,
                     1e20, -1e20, 0.5, -0.75], dtype=np.float32)
    for _ in range(50):
        q = _bf16(rng.choice(pool, size=d))
        kmin, kmax = _pages(rng, 64, d, pool)
        m, s = _sums(q, kmin, kmax)
        assert _same(m, s)


def test_negative_zero_query_takes_either_operand():
    # q = -0 selects kmin, q = +0 selects kmax: both products are zeros and
    # the sum is unchanged either way
    kmin = np.array([[-3.0, 1.0]], dtype=np.float32)
    kmax = np.array([[2.0, 5.0]], dtype=np.float32)
    for q in ([-0.0, 1.0], [0.0, 1.0], [-0.0, -0.0]):
        m, s = _sums(np.array(q, dtype=np.float32), kmin, kmax)
        assert _same(m, s)
