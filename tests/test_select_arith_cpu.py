"""The select pass's packed comparisons, emulated on the CPU.

Distances are u16 values 0 .. 384 G (at most 3072).  Two of them share a 32-bit word
(position 2j in the low half, 2j + 1 in the high half).  With c = (0x8000 + D*) * 0x10001,
the word c - w keeps bit 15 set iff the low distance is <= D* and bit 31 iff the high one
is, with no borrow between the halves; c - 0x10001 gives "< D*" the same way.  A byte
permute (selector 0x7531) gathers the high bytes of two such words and one multiply by
0x00204081 moves their four top bits to bits 28 .. 31 in position order.  This restates
those steps on integers and checks them against plain comparisons."""
import numpy as np

M = 0xFFFFFFFF


def _byte_perm(x, y, s):
    b = [(x >> (8 * i)) & 255 for i in range(4)] + [(y >> (8 * i)) & 255 for i in range(4)]
    return sum(b[(s >> (4 * i)) & 7] << (8 * i) for i in range(4))


def _lane_sign_bits(w0, w1):
    b = _byte_perm(w0, w1, 0x7531) & 0x80808080
    return ((b * 0x00204081) & M) >> 28


def _word(lo, hi):
    return (lo | (hi << 16)) & M


def test_packed_compare_all_distances():
    rng = np.random.default_rng(2)
    for dstar in [0, 1, 2, 127, 383, 384, 1535, 3071, 3072] + list(rng.integers(0, 3073, 8)):
        cle = ((0x8000 + int(dstar)) * 0x10001) & M
        clt = (cle - 0x10001) & M
        lo = rng.integers(0, 3073, 4000)
        hi = rng.integers(0, 3073, 4000)
        for a, b in zip(lo.tolist() + [0, 3072, int(dstar)], hi.tolist() + [3072, 0, int(dstar)]):
            w = _word(a, b)
            le, lt = (cle - w) & M, (clt - w) & M
            assert bool(le >> 15 & 1) == (a <= dstar) and bool(le >> 31 & 1) == (b <= dstar)
            assert bool(lt >> 15 & 1) == (a < dstar) and bool(lt >> 31 & 1) == (b < dstar)


def test_lane_sign_bits_in_position_order():
    for bits in range(16):
        # four 16-bit lanes (positions 0..3) with bit 15 set where `bits` says
        lanes = [(0x8000 if bits >> i & 1 else 0) | (0x1234 & 0x7FFF) for i in range(4)]
        w0, w1 = _word(lanes[0], lanes[1]), _word(lanes[2], lanes[3])
        assert _lane_sign_bits(w0, w1) == bits


def test_eight_positions_mask_matches_comparisons():
    rng = np.random.default_rng(7)
    for _ in range(2000):
        dstar = int(rng.integers(0, 3073))
        d = rng.integers(0, 3073, 8).tolist()
        cle = ((0x8000 + dstar) * 0x10001) & M
        clt = (cle - 0x10001) & M
        v = [_word(d[2 * j], d[2 * j + 1]) for j in range(4)]
        l0 = _lane_sign_bits((clt - v[0]) & M, (clt - v[1]) & M)
        l1 = _lane_sign_bits((clt - v[2]) & M, (clt - v[3]) & M)
        e0 = _lane_sign_bits((cle - v[0]) & M, (cle - v[1]) & M) & ~l0 & 0xF
        e1 = _lane_sign_bits((cle - v[2]) & M, (cle - v[3]) & M) & ~l1 & 0xF
        ltm, eqm = l0 | (l1 << 4), e0 | (e1 << 4)
        assert ltm == sum(1 << i for i in range(8) if d[i] < dstar)
        assert eqm == sum(1 << i for i in range(8) if d[i] == dstar)
