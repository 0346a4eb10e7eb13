"""Pins for the CPU oracle, each independent of the oracle's own code.

* packing: Python's own base-4 / base-3 number conversion, exhaustive over the
  byte and word patterns that matter;
* dequant + product: a second implementation with exact rationals
  (fractions.Fraction) written from the definition, per output element,
  without a dense W or a matmul;
* the add/subtract identity for ternary weights (promptzone article, "What It
  Is and How It Works": with weights in {-1, 0, +1} the product is additions and
  subtractions of activations);
* closed-form special cases (zero plane, single nonzero, all +1, r = N);
* planted mistakes: variants of the oracle with a plausible bug each (a
  dropped residual term, a transposed scale index, a wrong group width, a
  flipped sign, an off-by-one residual slot) must all fail the rational check.
"""

import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import tern_oracle as O
from ternary_weight_only_tern_b200 import synth


# ----------------------------------------------------------------------------- packing

def test_pack_exec_matches_python_base4():
    rng = np.random.default_rng(11)
    t = rng.integers(-1, 2, size=(7, 64)).astype(np.int8)
    words, bad = oracle.pack_exec(t)
    assert bad == 0 and words.shape == (7, 4) and words.dtype == np.uint32
    for r in range(7):
        for w in range(4):
            codes = [int(v) + 1 for v in t[r, 16 * w:16 * w + 16]]
            # code of trit k is base-4 digit k (least significant first)
            expect = int("".join(str(c) for c in reversed(codes)), 4)
            assert int(words[r, w]) == expect


def test_unpack_exec_every_byte_pattern():
    # all 256 byte values at each of the four byte positions of a word
    vals = np.arange(256, dtype=np.uint32)
    for pos in range(4):
        words = (vals << np.uint32(8 * pos)) | np.uint32(0x55555555 & ~(0xFF << (8 * pos)))
        t, bad = oracle.unpack_exec(words.reshape(256, 1), 16)
        n_bad = 0
        for v in range(256):
            digits = [int(d) for d in reversed(np.base_repr(v, 4).zfill(4))]
            for i, d in enumerate(digits):
                k = 4 * pos + i
                if d == 3:
                    n_bad += 1
                    assert t[v, k] == 0
                else:
                    assert t[v, k] == d - 1
            others = [k for k in range(16) if not (4 * pos <= k < 4 * pos + 4)]
            assert (t[v, others] == 0).all()     # code 1 elsewhere is trit 0
        # each of the 4 digits is 3 in 64 of the 256 bytes; 3**4 = 81 bytes hold no 3 at all
        assert bad == n_bad == 4 * 64
        assert sum(1 for v in range(256) if '3' not in np.base_repr(v, 4)) == 81


def test_pack_store_exhaustive_243():
    combos = np.array(np.meshgrid(*[np.arange(-1, 2)] * 5, indexing="ij")).reshape(5, -1).T.astype(np.int8)
    assert combos.shape == (243, 5)
    b, bad = oracle.pack_store(combos)
    assert bad == 0 and b.shape == (243, 1)
    for row, trits in zip(b[:, 0], combos):
        expect = int("".join(str(int(v) + 1) for v in reversed(trits)), 3)
        assert int(row) == expect
    assert sorted(int(v) for v in b[:, 0]) == list(range(243))   # a bijection onto 0..242
    t, bad = oracle.unpack_store(b, 5)
    assert bad == 0 and np.array_equal(t, combos)


def test_unpack_store_rejects_high_bytes():
    b = np.arange(256, dtype=np.uint8).reshape(256, 1)
    t, bad = oracle.unpack_store(b, 5)
    assert bad == 13
    assert (t[243:] == 0).all()
    for v in range(243):
        digits = [int(d) for d in reversed(np.base_repr(v, 3).zfill(5))]
        assert list(t[v]) == [d - 1 for d in digits]


@pytest.mark.parametrize("K", [1, 4, 5, 6, 127, 128, 2560, 2563])
def test_store_padding_and_roundtrip(K):
    rng = np.random.default_rng(K)
    t = rng.integers(-1, 2, size=(5, K)).astype(np.int8)
    b, bad = oracle.pack_store(t)
    assert bad == 0 and b.shape == (5, -(-K // 5))
    back, bad = oracle.unpack_store(b, K)
    assert bad == 0 and np.array_equal(back, t)
    if K % 5:
        # the padding digits of the last byte are 1 (trit 0): the last byte's value is below 3**(K%5) * ... +
        last = b[:, -1].astype(int)
        tail = K % 5
        assert all(v // 3 ** tail == sum(3 ** i for i in range(5 - tail)) for v in last)
        # a non-canonical padding digit is reported
        bb = b.copy()
        bb[0, -1] = int(bb[0, -1]) - 3 ** tail if bb[0, -1] >= 3 ** tail else int(bb[0, -1]) + 3 ** tail
        _, bad = oracle.unpack_store(bb, K)
        assert bad == 1


def test_exec_roundtrip_and_invalid_trits():
    rng = np.random.default_rng(3)
    t = rng.integers(-1, 2, size=(9, 256)).astype(np.int8)
    w, bad = oracle.pack_exec(t)
    back, bad2 = oracle.unpack_exec(w, 256)
    assert bad == bad2 == 0 and np.array_equal(back, t)
    t2 = t.copy()
    t2[0, 5] = 2
    t2[3, 17] = -7
    w2, bad = oracle.pack_exec(t2)
    assert bad == 2
    back, _ = oracle.unpack_exec(w2, 256)
    assert back[0, 5] == 0 and back[3, 17] == 0


# ----------------------------------------------------------------------------- linear

def brute_linear(x, T1, s1, res_rows, T2, s2, mu=None, elem=None):
    """Exact rational y[m][n] = sum_k x[m,k] * (mu[n,k//128] + s1[n,k//128] T1[n,k]
    + [n in R] s2[rho(n),k//128] T2[rho(n),k] + s2e[n,k//128] T2e[n,k]) (mu, elem absent: 0)."""
    M, K = x.shape
    N = T1.shape[0]
    rho = {int(n): i for i, n in enumerate(res_rows)}
    y = [[Fraction(0)] * N for _ in range(M)]
    for m in range(M):
        for n in range(N):
            acc = Fraction(0)
            for k in range(K):
                g = k // 128
                w = Fraction(float(s1[n][g])) * int(T1[n][k])
                if mu is not None:
                    w += Fraction(float(mu[n][g]))
                if n in rho:
                    w += Fraction(float(s2[rho[n]][g])) * int(T2[rho[n]][k])
                if elem is not None:
                    w += Fraction(float(elem[1][n][g])) * int(elem[0][n][k])
                acc += Fraction(float(x[m][k])) * w
            y[m][n] = acc
    return y


def check_against_brute(lin, case):
    x, T1, s1, rr, T2, s2 = case
    y = lin(x, T1, s1, rr, T2, s2)
    yb = brute_linear(x, T1, s1, rr, T2, s2)
    M, N = y.shape
    for m in range(M):
        for n in range(N):
            scale = sum(abs(float(x[m][k])) for k in range(x.shape[1])) * 0.05 + 1e-30
            if abs(Fraction(float(y[m, n])) - yb[m][n]) > Fraction(scale * 1e-14):
                return False
    return True


def tiny_cases():
    rng = np.random.default_rng(2024)
    cases = []
    for (N, K, M, r) in [(5, 128, 1, 2), (8, 256, 3, 3), (6, 256, 2, 6), (7, 128, 2, 0)]:
        t = synth.draw_tensor(rng, "tiny", N, K, M, p_zero=0.4, res_pct=0)
        res_rows = np.sort(rng.choice(N, size=r, replace=False)).astype(np.int32)
        T2 = synth.draw_trits(rng, (r, K), 0.4)
        s2 = synth.draw_scales(rng, r, K, 0.001, 0.005)
        cases.append((t.x, t.T1, t.s1, res_rows, T2, s2))
    return cases


@pytest.mark.parametrize("idx", range(4))
def test_linear_matches_exact_rationals(idx):
    assert check_against_brute(oracle.linear, tiny_cases()[idx])


def test_dequant_matches_definition_elementwise():
    x, T1, s1, rr, T2, s2 = tiny_cases()[1]
    W = oracle.dequant(T1, s1, rr, T2, s2)
    rho = {int(n): i for i, n in enumerate(rr)}
    for n in range(T1.shape[0]):
        for k in range(T1.shape[1]):
            w = float(s1[n, k // 128]) * int(T1[n, k])
            if n in rho:
                w += float(s2[rho[n], k // 128]) * int(T2[rho[n], k])
            assert W[n, k] == w


def test_add_subtract_identity():
    rng = np.random.default_rng(5)
    N, K, M = 16, 384, 4
    x = rng.integers(-20, 21, size=(M, K)).astype(np.float16)      # integer x: both sides exact
    T1 = synth.draw_trits(rng, (N, K), 0.4)
    s1 = np.ones((N, K // 128), dtype=np.float16)
    y = oracle.linear(x, T1, s1, np.zeros(0, np.int32), np.zeros((0, K), np.int8), np.zeros((0, K // 128), np.float16))
    xf = x.astype(np.float64)
    for m in range(M):
        for n in range(N):
            plus = xf[m][T1[n] == 1].sum()
            minus = xf[m][T1[n] == -1].sum()
            assert y[m, n] == plus - minus


def test_special_cases():
    rng = np.random.default_rng(9)
    N, K, M = 8, 256, 2
    x = synth.draw_x(rng, M, K)
    s1 = synth.draw_scales(rng, N, K, 0.005, 0.02)
    none_r = np.zeros(0, np.int32)
    z2 = np.zeros((0, K), np.int8)
    zs = np.zeros((0, K // 128), np.float16)
    # zero plane -> zero output
    assert (oracle.linear(x, np.zeros((N, K), np.int8), s1, none_r, z2, zs) == 0).all()
    # one nonzero per row -> +-s*x_k exactly
    T = np.zeros((N, K), np.int8)
    ks = rng.integers(0, K, size=N)
    sg = rng.choice([-1, 1], size=N)
    T[np.arange(N), ks] = sg
    y = oracle.linear(x, T, s1, none_r, z2, zs)
    for n in range(N):
        for m in range(M):
            assert y[m, n] == sg[n] * float(s1[n, ks[n] // 128]) * float(x[m, ks[n]])
    # all +1 -> sum over groups of s * (sum of x in the group)
    y = oracle.linear(x, np.ones((N, K), np.int8), s1, none_r, z2, zs)
    gx = x.astype(np.float64).reshape(M, K // 128, 128).sum(axis=2)
    assert np.allclose(y, gx @ s1.astype(np.float64).T, rtol=1e-13, atol=1e-13)
    # r = N with T2 = T1, s2 = s1 doubles the output; r = 0 leaves it alone
    T1 = synth.draw_trits(rng, (N, K), 0.4)
    y1 = oracle.linear(x, T1, s1, none_r, z2, zs)
    y2 = oracle.linear(x, T1, s1, np.arange(N, dtype=np.int32), T1, s1)
    assert np.allclose(y2, 2 * y1, rtol=1e-13, atol=1e-13)


def test_sampled_columns_match_full():
    rng = np.random.default_rng(1)
    t = synth.draw_tensor(rng, "s", 40, 256, 3, p_zero=0.4, res_pct=25)
    full = oracle.linear(t.x, t.T1, t.s1, t.res_rows, t.T2, t.s2)
    cols = np.array([0, 3, 17, 39, int(t.res_rows[0])])
    part = oracle.linear(t.x, t.T1, t.s1, t.res_rows, t.T2, t.s2, cols=cols)
    assert np.array_equal(part, full[:, cols])


# ------------------------------------------------------------------ planted mistakes

def _mut_drop_residual(x, T1, s1, rr, T2, s2):
    return O.linear(x, T1, s1, np.zeros(0, np.int32), T2[:0], s2[:0])


def _mut_scale_index(x, T1, s1, rr, T2, s2):
    # scale indexed by k % G instead of k // 128 (a transposed/misread index)
    N, K = T1.shape
    G = K // 128
    idx = np.arange(K) % G
    W = s1.astype(np.float64)[:, idx] * T1
    if len(rr):
        W[rr] += s2.astype(np.float64)[:, idx] * T2
    return x.astype(np.float64) @ W.T


def _mut_group_width(x, T1, s1, rr, T2, s2):
    N, K = T1.shape
    idx = np.minimum(np.arange(K) // 64, K // 128 - 1)
    W = s1.astype(np.float64)[:, idx] * T1
    if len(rr):
        W[rr] += s2.astype(np.float64)[:, idx] * T2
    return x.astype(np.float64) @ W.T


def _mut_sign(x, T1, s1, rr, T2, s2):
    W = O.dequant(T1, s1, rr, T2, s2)
    if len(rr):
        W[rr] -= 2 * np.repeat(s2.astype(np.float64), 128, axis=1) * T2
    return x.astype(np.float64) @ W.T


def _mut_slot_shift(x, T1, s1, rr, T2, s2):
    if len(rr) < 2:
        return O.linear(x, T1, s1, rr, T2, s2) + 1.0
    return O.linear(x, T1, s1, rr, np.roll(T2, 1, axis=0), np.roll(s2, 1, axis=0))


@pytest.mark.parametrize("mutant", [_mut_drop_residual, _mut_scale_index, _mut_group_width, _mut_sign,
                                    _mut_slot_shift])
def test_planted_mistakes_are_caught(mutant):
    cases = tiny_cases()
    assert not all(check_against_brute(mutant, c) for c in cases[:3])


# ----------------------------------------------------------------------------- exact case

def test_exact_inputs_are_exact_in_fp32_sums():
    rng = np.random.default_rng(4)
    t = synth.draw_exact_tensor(rng, 12, 512, 3, 4)
    y = oracle.linear(t.x, t.T1, t.s1, t.res_rows, t.T2, t.s2)
    yb = brute_linear(t.x, t.T1, t.s1, t.res_rows, t.T2, t.s2)
    for m in range(3):
        for n in range(12):
            assert Fraction(float(y[m, n])) == yb[m][n]                # float64 exact
            assert (yb[m][n] * 64).denominator == 1                    # multiple of 2^-6
            assert abs(yb[m][n]) < 2 ** 18
    # s1*t1 + s2*t2 exact in fp16
    W = oracle.dequant(t.T1, t.s1, t.res_rows, t.T2, t.s2)
    assert np.array_equal(W.astype(np.float16).astype(np.float64), W)


def test_round_fp16_is_round_to_nearest_even():
    # 1 + 2^-11 is halfway between 1 and the next fp16 (1 + 2^-10): ties to even -> 1
    assert float(oracle.round_fp16(np.array([1 + 2 ** -11]))[0]) == 1.0
    assert float(oracle.round_fp16(np.array([1 + 3 * 2 ** -11]))[0]) == 1 + 2 ** -9
    assert float(oracle.round_fp16(np.array([1 + 2 ** -11 + 2 ** -30]))[0]) == 1 + 2 ** -10


def test_rel_err():
    assert oracle.rel_err(np.array([1.0, 2.0]), np.array([1.0, 2.0])) == 0.0
    assert math.isclose(oracle.rel_err(np.array([1.0, 2.002]), np.array([1.0, 2.0])), 0.001)


# ---------------------------------------------------------------------- per-group offset mu
def offset_cases():
    rng = np.random.default_rng(77)
    out = []
    for (N, K, M, r) in [(5, 128, 2, 2), (6, 256, 1, 0), (4, 256, 3, 4)]:
        x = synth.draw_x(rng, M, K)
        T1 = synth.draw_trits(rng, (N, K), 0.4)
        s1 = synth.draw_scales(rng, N, K, 0.005, 0.02)
        rr = np.sort(rng.choice(N, size=r, replace=False)).astype(np.int32)
        T2 = synth.draw_trits(rng, (r, K), 0.4)
        s2 = synth.draw_scales(rng, r, K, 0.001, 0.005)
        mu = (rng.uniform(-0.01, 0.01, size=(N, K // 128))).astype(np.float16)
        out.append((x, T1, s1, rr, T2, s2, mu))
    return out


@pytest.mark.parametrize("idx", range(3))
def test_offset_matches_exact_rationals(idx):
    x, T1, s1, rr, T2, s2, mu = offset_cases()[idx]
    y = oracle.linear(x, T1, s1, rr, T2, s2, mu=mu)
    yb = brute_linear(x, T1, s1, rr, T2, s2, mu=mu)
    for m in range(y.shape[0]):
        for n in range(y.shape[1]):
            scale = sum(abs(float(v)) for v in x[m]) * 0.05 + 1e-30
            assert abs(Fraction(float(y[m, n])) - yb[m][n]) <= Fraction(scale * 1e-14)


def test_constant_offset_shifts_every_row_by_the_activation_sum():
    """mu = c everywhere adds c * sum_k x[m, k] to every output of token m."""
    x, T1, s1, rr, T2, s2, mu = offset_cases()[2]
    c = np.float16(0.0078125)
    y0 = oracle.linear(x, T1, s1, rr, T2, s2)
    y1 = oracle.linear(x, T1, s1, rr, T2, s2, mu=np.full_like(mu, c))
    shift = float(c) * x.astype(np.float64).sum(axis=1)
    np.testing.assert_allclose(y1 - y0, np.repeat(shift[:, None], y0.shape[1], axis=1), rtol=1e-12, atol=1e-15)


def test_offset_alone_is_the_scaled_group_sums():
    """Zero planes: y[m, n] = sum_g mu[n, g] * (sum of x[m] over group g), group sums by Python loops."""
    x, T1, s1, rr, T2, s2, mu = offset_cases()[0]
    Z1, Z2 = np.zeros_like(T1), np.zeros_like(T2)
    y = oracle.linear(x, Z1, s1, rr, Z2, s2, mu=mu)
    M, K = x.shape
    for m in range(M):
        sums = [sum(float(x[m, k]) for k in range(g * 128, (g + 1) * 128)) for g in range(K // 128)]
        for n in range(mu.shape[0]):
            assert y[m, n] == pytest.approx(sum(float(mu[n, g]) * sums[g] for g in range(K // 128)), rel=1e-12)


def test_planted_offset_mistake_is_caught():
    """An oracle that adds the offset of the wrong group fails the rational check."""
    x, T1, s1, rr, T2, s2, mu = offset_cases()[1]
    bad = oracle.linear(x, T1, s1, rr, T2, s2, mu=np.roll(mu, 1, axis=1))
    yb = brute_linear(x, T1, s1, rr, T2, s2, mu=mu)
    assert any(abs(Fraction(float(bad[m, n])) - yb[m][n]) > Fraction(1e-9)
               for m in range(bad.shape[0]) for n in range(bad.shape[1]))



# ---------------------------------------------------------------- element-level second plane
def hand_elem():
    """N = 2, K = 256. Nonzero T2e: row 0: k=3 -> +1, k=130 -> -1; row 1: k=0 -> -1,
    k=127 -> +1, k=255 -> +1. Worked by hand: group 0 lists row 0 (3 << 1 = 6), then row 1
    (0 << 1 | 1 = 1, 127 << 1 = 254); group 1 lists row 0 (2 << 1 | 1 = 5), then row 1
    (127 << 1 = 254). ecount[g][n] = [[1, 2], [1, 1]]; one 64-row block per group, so
    ebase = [0, 3, 5]."""
    T = np.zeros((2, 256), np.int8)
    T[0, 3], T[0, 130], T[1, 0], T[1, 127], T[1, 255] = 1, -1, -1, 1, 1
    return T, np.array([[1, 2], [1, 1]], np.uint8), np.array([0, 3, 5]), np.array([6, 1, 254, 5, 254], np.uint8)


def test_pack_elem_hand_worked_example():
    T, cnt, base, idx = hand_elem()
    c, b, e, bad = oracle.pack_elem(T)
    assert bad == 0
    assert np.array_equal(c, cnt) and np.array_equal(b, base) and np.array_equal(e, idx)
    T2, bad2 = oracle.unpack_elem(cnt, base, idx, 2, 256)
    assert bad2 == 0 and np.array_equal(T2, T)


def _elem_mut_sign(T):
    c, b, e, _ = oracle.pack_elem(T)
    return c, b, e ^ np.uint8(1)


def _elem_mut_no_shift(T):
    c, b, e, _ = oracle.pack_elem(T)
    return c, b, (e >> 1).astype(np.uint8)


def _elem_mut_row_major(T):
    # rows first, then groups: the order of the entries is wrong
    N, K = T.shape
    out = [int(kk) << 1 | int(T[n, g * 128 + kk] < 0) for n in range(N) for g in range(K // 128)
           for kk in np.flatnonzero(T[n, g * 128:(g + 1) * 128])]
    c, b, _, _ = oracle.pack_elem(T)
    return c, b, np.array(out, np.uint8)


@pytest.mark.parametrize("mutant", [_elem_mut_sign, _elem_mut_no_shift, _elem_mut_row_major])
def test_planted_elem_packing_mistakes_are_caught(mutant):
    T, cnt, base, idx = hand_elem()
    c, b, e = mutant(T)
    assert not (np.array_equal(c, cnt) and np.array_equal(b, base) and np.array_equal(e, idx))


@pytest.mark.parametrize("N,K,density", [(1, 128, 0.05), (63, 256, 0.03), (64, 128, 0.0), (65, 384, 0.03),
                                         (130, 128, 1.0), (200, 256, 0.2)])
def test_elem_roundtrip_and_counts(N, K, density):
    rng = np.random.default_rng(N * K)
    T = np.where(rng.random((N, K)) < density, rng.choice(np.array([-1, 1], np.int8), (N, K)), 0).astype(np.int8)
    c, b, e, bad = oracle.pack_elem(T)
    assert bad == 0 and len(e) == np.count_nonzero(T) and int(b[-1]) == len(e)
    G, NB = K // 128, oracle.elem_blocks(N)
    for g in range(G):                      # counts are the nonzeros of each (row, group), by numpy
        assert np.array_equal(c[g], np.count_nonzero(T[:, g * 128:(g + 1) * 128], axis=1))
    assert np.all(np.diff(b) >= 0) and b.shape == (G * NB + 1,)
    T2, bad2 = oracle.unpack_elem(c, b, e, N, K)
    assert bad2 == 0 and np.array_equal(T2, T)


def test_pack_elem_counts_invalid_trits():
    T = np.zeros((3, 128), np.int8)
    T[0, 5], T[1, 9], T[2, 0] = 2, -7, 1
    c, b, e, bad = oracle.pack_elem(T)
    assert bad == 2 and list(e) == [0] and list(c[0]) == [0, 0, 1]


def test_unpack_elem_flags_inconsistent_metadata():
    T, cnt, base, idx = hand_elem()
    assert oracle.unpack_elem(cnt, base, idx[[0, 2, 1, 3, 4]], 2, 256)[1] > 0     # k not increasing
    c2 = cnt.copy(); c2[0, 1] = 1
    assert oracle.unpack_elem(c2, base, idx, 2, 256)[1] > 0                      # block sum != base gap
    assert oracle.unpack_elem(cnt, np.array([1, 3, 5]), idx, 2, 256)[1] > 0      # ebase[0] != 0
    assert oracle.unpack_elem(cnt, base, idx[:4], 2, 256)[1] > 0                 # last base != nnz2
    c3 = cnt.copy(); c3[0, 0] = 200
    assert oracle.unpack_elem(c3, base, idx, 2, 256)[1] > 0                      # count above 128


def elem_cases():
    rng = np.random.default_rng(91)
    out = []
    for (N, K, M, r) in [(5, 128, 2, 0), (4, 256, 2, 2), (3, 256, 1, 0)]:
        x = synth.draw_x(rng, M, K)
        T1 = synth.draw_trits(rng, (N, K), 0.4)
        s1 = synth.draw_scales(rng, N, K, 0.005, 0.02)
        rr = np.sort(rng.choice(N, size=r, replace=False)).astype(np.int32)
        T2 = synth.draw_trits(rng, (r, K), 0.4)
        s2 = synth.draw_scales(rng, r, K, 0.001, 0.005)
        T2e = np.where(rng.random((N, K)) < 0.1, synth.draw_trits(rng, (N, K), 0.4), 0).astype(np.int8)
        s2e = synth.draw_scales(rng, N, K, 0.001, 0.005)
        out.append((x, T1, s1, rr, T2, s2, (T2e, s2e)))
    return out


@pytest.mark.parametrize("idx", range(3))
def test_elem_plane_matches_exact_rationals(idx):
    x, T1, s1, rr, T2, s2, elem = elem_cases()[idx]
    y = oracle.linear(x, T1, s1, rr, T2, s2, elem=elem)
    yb = brute_linear(x, T1, s1, rr, T2, s2, elem=elem)
    for m in range(y.shape[0]):
        for n in range(y.shape[1]):
            scale = sum(abs(float(v)) for v in x[m]) * 0.05 + 1e-30
            assert abs(Fraction(float(y[m, n])) - yb[m][n]) <= Fraction(scale * 1e-14)


def test_elem_plane_on_whole_rows_is_the_row_residual():
    """An element plane that covers whole rows R with T2e[R] = T2 and s2e[R] = s2 is the
    row-form residual: the two dequantised W are equal element for element."""
    rng = np.random.default_rng(5)
    N, K, r = 70, 384, 9
    T1 = synth.draw_trits(rng, (N, K), 0.4)
    s1 = synth.draw_scales(rng, N, K, 0.005, 0.02)
    rr = np.sort(rng.choice(N, size=r, replace=False)).astype(np.int32)
    T2 = synth.draw_trits(rng, (r, K), 0.4)
    s2 = synth.draw_scales(rng, r, K, 0.001, 0.005)
    T2e = np.zeros((N, K), np.int8)
    T2e[rr] = T2
    s2e = synth.draw_scales(rng, N, K, 0.001, 0.005)
    s2e[rr] = s2
    W_row = oracle.dequant(T1, s1, rr, T2, s2)
    W_elem = oracle.dequant(T1, s1, np.zeros(0, np.int32), np.zeros((0, K), np.int8),
                            np.zeros((0, K // 128), np.float16), elem=(T2e, s2e))
    assert np.array_equal(W_row, W_elem)


def test_planted_elem_scale_mistake_is_caught():
    """An oracle that takes the element plane's scale from the next row fails the rational check."""
    x, T1, s1, rr, T2, s2, (T2e, s2e) = elem_cases()[0]
    bad = oracle.linear(x, T1, s1, rr, T2, s2, elem=(T2e, np.roll(s2e, 1, axis=0)))
    yb = brute_linear(x, T1, s1, rr, T2, s2, elem=(T2e, s2e))
    assert any(abs(Fraction(float(bad[m, n])) - yb[m][n]) > Fraction(1e-9)
               for m in range(bad.shape[0]) for n in range(bad.shape[1]))



# ---------------------------------------------------------------- activation-side rotation
def _orthogonal_blocks(rng, G):
    """G random 128 x 128 orthogonal blocks (float64, QR of a Gaussian), not symmetric."""
    out = np.empty((G, 128, 128))
    for g in range(G):
        q, r = np.linalg.qr(rng.standard_normal((128, 128)))
        out[g] = q * np.sign(np.diag(r))
    return out


def test_rotate_by_identity_and_signed_permutations_is_exact():
    rng = np.random.default_rng(8)
    x = synth.draw_x(rng, 3, 384)
    eye = np.stack([np.eye(128)] * 3)
    assert np.array_equal(oracle.rotate(x, eye), x.astype(np.float64))
    # block g sends input i to output perm[g][i] with sign sgn[g][i]
    perm = [rng.permutation(128) for _ in range(3)]
    sgn = [rng.choice([-1.0, 1.0], 128) for _ in range(3)]
    R = np.zeros((3, 128, 128))
    for g in range(3):
        for i in range(128):
            R[g, i, perm[g][i]] = sgn[g][i]
    y = oracle.rotate(x, R)
    for m in range(3):
        for g in range(3):
            for i in range(128):
                assert y[m, g * 128 + perm[g][i]] == sgn[g][i] * float(x[m, g * 128 + i])


def test_rotate_matches_exact_rationals():
    rng = np.random.default_rng(9)
    x = synth.draw_x(rng, 2, 256)
    R = rng.integers(-3, 4, size=(2, 128, 128)).astype(np.float64) / 8
    y = oracle.rotate(x, R)
    for m in range(2):
        for g in range(2):
            for j in range(0, 128, 17):
                exact = sum(Fraction(float(x[m, g * 128 + i])) * Fraction(R[g, i, j]) for i in range(128))
                assert Fraction(float(y[m, g * 128 + j])) == exact


def test_rotated_activations_with_rotated_weights_give_the_layer():
    """x' = x R and W' = W R (R orthogonal, block-diagonal) give x' W'^T = x W^T: the rotation
    the pages apply to activations is the one that undoes the weights' basis change."""
    from scipy.linalg import block_diag
    rng = np.random.default_rng(10)
    N, K, M = 7, 384, 3
    x = synth.draw_x(rng, M, K)
    W = oracle.dequant(synth.draw_trits(rng, (N, K), 0.4), synth.draw_scales(rng, N, K, 0.005, 0.02),
                       np.zeros(0, np.int32), np.zeros((0, K), np.int8), np.zeros((0, 3), np.float16))
    blocks = _orthogonal_blocks(rng, 3)
    Rfull = block_diag(*blocks)
    y = oracle.rotate(x, blocks) @ (W @ Rfull).T
    np.testing.assert_allclose(y, x.astype(np.float64) @ W.T, rtol=0, atol=1e-12 * np.abs(W).sum())
    # planted mistake: the transposed blocks do not undo the basis change
    bad = oracle.rotate(x, np.transpose(blocks, (0, 2, 1))) @ (W @ Rfull).T
    assert np.abs(bad - x.astype(np.float64) @ W.T).max() > 1e-3



# ---------------------------------------------------------------- ternarization fit
def _hand_group():
    """64 entries of 1.0 and 64 of fp16(0.4), no offset. Worked by hand: mean |w| = (64 + 64 x 0.4)
    / 128 ~ 0.7, threshold 0.49: the first plane holds the ones (a1 = 1); its residual is 0.4 on
    the other half, mean 0.2, threshold 0.14: the second plane holds them (a2 = fp16(0.4)); the
    refinement keeps both, and mu + a1 T1 + a2 T2 = w exactly."""
    w = np.array([1.0] * 64 + [0.4] * 64, dtype=np.float16)
    return w, np.array([1] * 64 + [0] * 64, np.int8), np.array([0] * 64 + [1] * 64, np.int8)


def test_fit_hand_worked_group():
    w, t1, t2 = _hand_group()
    T1, a1, mu, T2, a2 = oracle.fit_groups(w.astype(np.float64)[None], np.array([True]), False, 15)
    assert np.array_equal(T1[0], t1) and np.array_equal(T2[0], t2)
    assert a1[0] == 1.0 and a2[0] == float(np.float16(0.4)) and mu[0] == 0.0


def test_planted_threshold_mistake_is_caught(monkeypatch):
    """A fit with the threshold at 0.5 mean |r| puts the 0.4 entries into the first plane."""
    w, t1, _ = _hand_group()
    monkeypatch.setattr(O, "TWN_RATIO", 0.5)
    T1, *_ = O.fit_groups(w.astype(np.float64)[None], np.array([True]), False, 15)
    assert not np.array_equal(T1[0], t1)


def test_fit_recovers_an_exactly_ternary_group_with_offset():
    rng = np.random.default_rng(12)
    t = np.array([-1] * 40 + [0] * 48 + [1] * 40, np.int8)
    rng.shuffle(t)
    w = (0.25 + 0.5 * t).astype(np.float16).astype(np.float64)
    T1, a1, mu, T2, a2 = oracle.fit_groups(w[None], np.array([False]), True, 15)
    assert np.array_equal(T1[0], t) and a1[0] == 0.5 and mu[0] == 0.25 and not T2.any() and a2[0] == 0.0


def test_refinement_reaches_least_squares_and_never_increases_the_error():
    rng = np.random.default_rng(13)
    w = (rng.standard_normal((6, 128)) * 0.02 + 0.003).astype(np.float16).astype(np.float64)
    has2 = np.array([True, False, True, True, False, True])
    errs = []
    for it in (0, 1, 2, 5, 15):
        T1, a1, mu, T2, a2 = oracle.fit_groups(w, has2, True, it)
        errs.append(((w - mu[:, None] - a1[:, None] * T1 - a2[:, None] * T2) ** 2).sum(axis=1))
    for e0, e1 in zip(errs, errs[1:]):
        assert np.all(e1 <= e0 * (1 + 1e-12) + 1e-300)
    T1, a1, mu, T2, a2 = oracle.fit_groups(w, has2, True, 400)
    for g in range(6):
        cols = [np.ones(128), T1[g].astype(np.float64)] + ([T2[g].astype(np.float64)] if has2[g] else [])
        sol = np.linalg.lstsq(np.stack(cols, axis=1), w[g], rcond=None)[0]
        assert abs(sol[0] - mu[g]) < 1e-9 and abs(sol[1] - a1[g]) < 1e-9
        if has2[g]:
            assert abs(sol[2] - a2[g]) < 1e-9


def test_fit_of_zero_and_constant_groups():
    w = np.stack([np.zeros(128), np.full(128, 0.125)])
    T1, a1, mu, T2, a2 = oracle.fit_groups(w, np.array([True, True]), True, 15)
    assert not T1.any() and not T2.any() and np.all(a1 == 0) and np.all(a2 == 0)
    assert mu[0] == 0 and mu[1] == 0.125


def test_ternarize_assembles_rows_and_groups():
    """ternarize is fit_groups over (row, group), with the second plane on the listed rows only."""
    rng = np.random.default_rng(14)
    W = (rng.standard_normal((9, 384)) * 0.02).astype(np.float16)
    rows = np.array([2, 5, 8])
    T1, s1, mu, T2, s2 = oracle.ternarize(W, rows)
    for n in range(9):
        for g in range(3):
            t1, a1, m, t2, a2 = oracle.fit_groups(W[n, g * 128:(g + 1) * 128].astype(np.float64)[None],
                                                  np.array([n in rows]), True, 15)
            assert np.array_equal(T1[n, g * 128:(g + 1) * 128], t1[0])
            assert s1[n, g] == np.float16(a1[0]) and mu[n, g] == np.float16(m[0])
            if n in rows:
                i = list(rows).index(n)
                assert np.array_equal(T2[i, g * 128:(g + 1) * 128], t2[0]) and s2[i, g] == np.float16(a2[0])


# ------------------------------------------------------------------ residual-row metadata
# The second plane lives on a sorted subset R of rows ("Post-Training Ternarization of
# Qwen3-4B", section 4.4; the 8B paper's representation paragraph). Its execution form is the
# slot map (row -> index in R, or -1), its storage form a bitmap of the rows.

def test_slot_map_and_bitmap_hand_worked():
    rows = np.array([1, 2, 9], np.int32)
    assert oracle.slot_map(11, rows).tolist() == [-1, 0, 1, -1, -1, -1, -1, -1, -1, 2, -1]
    # rows 1, 2 -> byte 0 = 0b00000110; row 9 -> byte 1 = 0b00000010
    assert oracle.row_bitmap(11, rows).tolist() == [6, 2]
    assert O.rows_from_bitmap(11, np.array([6, 2], np.uint8)).tolist() == [1, 2, 9]


@pytest.mark.parametrize("N", [1, 7, 8, 9, 63, 64, 65, 1000, 12288])
def test_residual_metadata_against_python_integers(N):
    rng = np.random.default_rng(N)
    for frac in (0.0, 0.15, 1.0):
        r = int(round(frac * N))
        rows = np.sort(rng.choice(N, size=r, replace=False)).astype(np.int32)
        # the bitmap is the little-endian bytes of the integer sum of 2^n over R
        as_int = sum(1 << int(n) for n in rows)
        want = np.frombuffer(as_int.to_bytes(-(-N // 8), "little"), dtype=np.uint8)
        assert np.array_equal(oracle.row_bitmap(N, rows), want)
        # the slot map, element by element from its definition
        slot = oracle.slot_map(N, rows)
        pos = {int(n): i for i, n in enumerate(rows)}
        assert all(int(slot[n]) == pos.get(n, -1) for n in range(N))
        assert np.array_equal(O.rows_from_bitmap(N, want), rows)


def test_rows_from_bitmap_ignores_bits_past_n():
    # byte 1 holds rows 8..15; with N = 10 only rows 8 and 9 exist
    assert O.rows_from_bitmap(10, np.array([0, 0xFF], np.uint8)).tolist() == [8, 9]
