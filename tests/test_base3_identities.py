"""The arithmetic the base-3 (1.6-bit) engines of the batch kernel and the
1.6-bit GEMM decode rest on, checked exhaustively on the CPU in Python
integers (the GPU parity tests then check the kernels themselves):

* floor(85 (v + 1) / 256) = floor(v / 3) for every valid code v < 243, and
  85 (v + 1) < 2^16 for every byte, so two bytes in 16-bit lanes of one
  32-bit register divide with one multiply-add and no carry between lanes;
  the quotient is the product's high byte (a PRMT moves it down);
* with q_p = floor(v / 3^p): sum_i d_i xi_i = q_0 xi_0 + sum_{p>=1} q_p
  (xi_p - 3 xi_{p-1}) (the telescoped activations of the integer engine);
* the integer engine's offsets: B_0 = xi_0 + 2^42, B_p = xi_p - 3 xi_{p-1} +
  2^42 lie in [0, 2^43) (six u8 planes) for |xi| < 2^40, and the plane
  sums weighted by 256^j, minus 2^42 times the ones column, give back the
  exact sum;
* the fp16 engine's digits d_p = E_p - 3 E_{p+1} per 16-bit lane never
  borrow across lanes.
"""
import random

MASK32 = 0xFFFFFFFF


def prmt(a, b, sel):
    """PTX prmt.b32 (default mode): byte i of the result is byte sel_i of b:a."""
    src = [(a >> (8 * i)) & 0xFF for i in range(4)] + [(b >> (8 * i)) & 0xFF for i in range(4)]
    return sum(src[(sel >> (4 * i)) & 7] << (8 * i) for i in range(4))


def digits(v):
    return [(v // 3 ** i) % 3 for i in range(5)]


def test_quotient_by_three_in_16_bit_lanes():
    for v in range(256):
        assert 85 * (v + 1) < 1 << 16
        if v < 243:
            assert (85 * (v + 1)) >> 8 == v // 3, v
    # the chain on packed words: lanes of even and odd bytes, quotient words
    rng = random.Random(5)
    for _ in range(3000):
        b = [rng.randrange(243) for _ in range(4)]
        w = b[0] | b[1] << 8 | b[2] << 16 | b[3] << 24
        E, O = prmt(w, 0, 0x4240), prmt(w, 0, 0x4341)
        for p in range(1, 5):
            tE = (E * 85 + 0x00550055) & MASK32
            tO = (O * 85 + 0x00550055) & MASK32
            P = prmt(tE, tO, 0x7351)  # the quotient word of the integer engine
            assert [(P >> (8 * e)) & 0xFF for e in range(4)] == [x // 3 ** p for x in b]
            E, O = prmt(tE, 0, 0x4341), prmt(tO, 0, 0x4341)


def test_digits_per_lane_never_borrow():
    # fp16 engine and GEMM: d = E - 3 E' per 16-bit lane
    for lo in range(243):
        for hi in (0, 1, 80, 121, 242):
            E = lo | hi << 16
            E1 = prmt((E * 85 + 0x00550055) & MASK32, 0, 0x4341)
            d = (E - 3 * E1) & MASK32
            assert d & 0xFFFF == lo % 3 and d >> 16 == hi % 3


def test_telescoped_sum_and_offsets():
    rng = random.Random(7)
    C = 1 << 42
    for v in range(243):
        d = digits(v)
        q = [v // 3 ** p for p in range(5)]
        for _ in range(20):
            xi = [rng.randrange(-(1 << 40) + 1, 1 << 40) for _ in range(5)]
            B = [xi[0] + C] + [xi[p] - 3 * xi[p - 1] + C for p in range(1, 5)]
            assert all(0 <= x < 1 << 43 for x in B)
            direct = sum(di * x for di, x in zip(d, xi))
            assert q[0] * xi[0] + sum(q[p] * (xi[p] - 3 * xi[p - 1]) for p in range(1, 5)) == direct
            # what the MMAs see: byte planes of B against the A bytes, and a ones column
            S = [sum(q[p] * ((B[p] >> (8 * j)) & 0xFF) for p in range(5)) for j in range(6)]
            ones = sum(q)
            assert sum(S[j] << (8 * j) for j in range(6)) - (ones << 42) == direct
