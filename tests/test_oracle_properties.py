"""Property tests of the oracle (hypothesis, CPU): round trips of the three packed forms and
relations the bit formulas must satisfy, on shapes and contents the generator chooses."""

import math

import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle

trit_arrays = st.integers(1, 5).flatmap(
    lambda rows: st.integers(1, 3).flatmap(
        lambda groups: st.lists(st.integers(-1, 1), min_size=rows * groups * 128, max_size=rows * groups * 128).map(
            lambda v: np.array(v, np.int8).reshape(rows, groups * 128))))


@settings(max_examples=40, deadline=None)
@given(trit_arrays)
def test_exec_and_store_round_trips(T):
    w, bad = oracle.pack_exec(T)
    assert bad == 0 and np.array_equal(oracle.unpack_exec(w, T.shape[1])[0], T)
    b, bad = oracle.pack_store(T)
    assert bad == 0 and np.array_equal(oracle.unpack_store(b, T.shape[1])[0], T)


@settings(max_examples=40, deadline=None)
@given(trit_arrays)
def test_elem_round_trip_and_sizes(T):
    c, b, e, bad = oracle.pack_elem(T)
    assert bad == 0
    assert len(e) == np.count_nonzero(T) and int(c.sum()) == len(e) and int(b[-1]) == len(e)
    T2, bad2 = oracle.unpack_elem(c, b, e, *T.shape)
    assert bad2 == 0 and np.array_equal(T2, T)
    # every listed byte names a position inside its group and a nonzero trit's sign
    assert np.all((e >> 1) < 128)


@settings(max_examples=60, deadline=None)
@given(st.integers(1, 10_000), st.integers(1, 64).map(lambda g: 128 * g), st.data())
def test_bit_formulas_relations(N, K, data):
    r = data.draw(st.integers(0, N))
    b = oracle.bits(N, K, r)
    # information rate log2(3) (1 + r/N), and each form above it
    assert math.isclose(b["bpw_info"], math.log2(3) * (1 + r / N), rel_tol=1e-12)
    assert b["bpw_exec"] > b["bpw_info"] and b["bpw_store"] > b["bpw_info"]
    # one more residual row adds exactly one row's bits to each form
    if r < N:
        b1 = oracle.bits(N, K, r + 1)
        G = K // 128
        assert b1["exec_bits"] - b["exec_bits"] == 2 * K + 16 * G
        assert b1["store_bits"] - b["store_bits"] == 8 * ((K + 4) // 5) + 16 * G
    # the offset adds 16 bits per (row, group); the element form with nothing masked is the
    # one-plane form plus its (empty) element arrays
    assert oracle.bits(N, K, r, offset=True)["exec_bits"] - b["exec_bits"] == 16 * N * (K // 128)
    e0 = oracle.bits_elem(N, K, 0, 0)
    one = oracle.bits(N, K, 0)
    G, NB = K // 128, -(-N // 64)
    assert e0["exec_bits"] - (one["exec_bits"] - 32 * N) == 8 * G * N + 32 * (G * NB + 1) + 16 * N * G


@settings(max_examples=25, deadline=None)
@given(st.integers(1, 4), st.integers(1, 3), st.integers(0, 2**32 - 1))
def test_fit_reconstruction_never_worse_than_zero(rows, groups, seed):
    """The fitted reconstruction is never farther from W than W itself is from zero (the fit
    can always fall back to an empty support)."""
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((rows, groups * 128)) * rng.uniform(1e-3, 1.0)).astype(np.float16)
    T1, s1, mu, T2, s2 = oracle.ternarize(W, np.arange(rows)[: rows // 2])
    Wh = oracle.dequant(T1, s1, np.arange(rows)[: rows // 2], T2, s2, mu=mu)
    Wd = W.astype(np.float64)
    assert np.linalg.norm(Wh - Wd) <= np.linalg.norm(Wd) * (1 + 1e-3)
