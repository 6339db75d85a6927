"""The packed form of the StatePassing link (eq. 6 of the SSDi8 notes) on CPU, exhaustively.

The W8A8 kernels carry H' = sat127(S + ((dq*H + 2^(k-1)) >> k)) on two codes per 32-bit
word: with Hu = H + 128 and Su = S + 128 in 16-bit fields,
    V = dq*Hu + 2^(k-1) + 128*(2^k - dq) + Su*2^k = dq*H + 2^(k-1) + (S + 256)*2^k,
which lies in [0, 2^16) for k <= 7 and 0 <= dq <= 2^k, so the fields never carry into each
other; V >> k is H' + 256 before saturation, so clamping each field to
[129*2^k, 384*2^k - 1] (unsigned 16-bit min/max) saturates, and the low byte of each
field after the word-wide shift by k is H' as an int8 code (bits shifted down from the
upper field land at bit 16 - k >= 9 of the lower one, above its low byte).

This test emulates that word arithmetic in 32-bit integers for every k in 1..7, every dq
in [0, 2^k] and every (H, S) pair of codes, with the other field holding every code pair
of a second sweep, and compares each byte with the plain rule.
"""
import numpy as np
import pytest

M32 = np.uint64(0xFFFFFFFF)


def _rule(h, s, dq, k):
    return np.clip(s + ((dq * h + (1 << (k - 1))) >> k), -127, 127)


def _field_clamp(v, lo, hi):
    f0, f1 = v & 0xFFFF, (v >> 16) & 0xFFFF
    f0 = np.minimum(np.maximum(f0, lo), hi)
    f1 = np.minimum(np.maximum(f1, lo), hi)
    return f0 | (f1 << 16)


def _packed(h0, s0, h1, s1, dq, k):
    """One 32-bit word: codes (h0, s0) in the low field, (h1, s1) in the high field."""
    hu = (h0 + 128) | ((h1 + 128) << 16)
    su = (s0 + 128) | ((s1 + 128) << 16)
    k0 = (1 << (k - 1)) + 128 * ((1 << k) - dq)
    v = (hu * dq + (k0 | (k0 << 16)) + (su << k)) & 0xFFFFFFFF
    v = _field_clamp(v, 129 << k, (384 << k) - 1) >> k
    b0, b1 = v & 0xFF, (v >> 16) & 0xFF
    return np.where(b0 > 127, b0 - 256, b0), np.where(b1 > 127, b1 - 256, b1)


@pytest.mark.parametrize("k", range(1, 8))
def test_packed_link_equals_the_rule_exhaustively(k):
    codes = np.arange(-127, 128, dtype=np.int64)
    h, s = np.meshgrid(codes, codes, indexing="ij")
    h, s = h.ravel(), s.ravel()
    # companion field: the same sweep reversed, so every pair meets many different neighbours
    h1, s1 = h[::-1].copy(), s[::-1].copy()
    for dq in range(0, (1 << k) + 1):
        got0, got1 = _packed(h, s, h1, s1, dq, k)
        np.testing.assert_array_equal(got0, _rule(h, s, dq, k), err_msg=f"low field k={k} dq={dq}")
        np.testing.assert_array_equal(got1, _rule(h1, s1, dq, k), err_msg=f"high field k={k} dq={dq}")


def test_packed_word_stays_below_two_to_the_sixteen():
    """The largest V (H = S = 127, dq = 2^k) fits a 16-bit field for k <= 7 and not for k = 8."""
    for k in range(1, 9):
        dq = 1 << k
        v = dq * 255 + (1 << (k - 1)) + 128 * ((1 << k) - dq) + 255 * (1 << k)
        assert (v < (1 << 16)) == (k <= 7), (k, v)
