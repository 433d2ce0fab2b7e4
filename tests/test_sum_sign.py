"""The branch-free weighted sum of combine forward adds w * 0 for a skipped or
zero-expert pair instead of leaving the pair out. That is exact because an
IEEE round-to-nearest sum that starts at +0 is never -0 (x + y is -0 only when
both are -0), and adding +0 or -0 to any other value leaves it unchanged. This
checks both facts in float32 on values chosen to reach exact cancellation,
signed zeros and the subnormal range."""
import itertools

import numpy as np


def _values():
    tiny = np.float32(np.finfo(np.float32).smallest_subnormal)
    base = [0.0, -0.0, 1.0, -1.0, 3.5, -3.5, 1e-30, -1e-30, 6.5e4, -6.5e4]
    vals = [np.float32(v) for v in base] + [tiny, -tiny, np.float32(2) * tiny, -np.float32(2) * tiny]
    return vals


def test_a_sum_from_plus_zero_is_never_minus_zero():
    vals = _values()
    for seq in itertools.product(vals, repeat=3):
        acc = np.float32(0.0)
        for x in seq:
            acc = np.float32(acc + x)
            assert not (acc == 0 and np.signbit(acc)), seq


def test_adding_a_signed_zero_leaves_a_non_minus_zero_sum_unchanged():
    vals = [v for v in _values() if not (v == 0 and np.signbit(v))]
    for acc, z in itertools.product(vals, (np.float32(0.0), np.float32(-0.0))):
        out = np.float32(acc + z)
        assert out.tobytes() == np.float32(acc).tobytes(), (acc, z)
    # the products a skipped pair adds: 0 * 0, and w * 0 for any finite weight
    for w in _values():
        p = np.float32(w * np.float32(0.0))
        assert p == 0
        for acc in vals:
            assert np.float32(acc + p).tobytes() == np.float32(acc).tobytes()
