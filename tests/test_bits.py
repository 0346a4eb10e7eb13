"""Pins for the bit accounting (oracle side; the C-ABI's tern_bits is compared in test_abi).

* the page figures (tests/golden/page_figures.json): the ideal rate log2 3 and the
  measured 1.641 / 1.64 bits per weight at the second-plane fraction the pages print;
* byte counting: the store and exec bit totals equal the sizes of arrays actually
  serialised with the oracle's packers;
* worked values for three shapes, reproduced as integers.
"""

import json
import math
import os

import numpy as np
import pytest

import oracle
from ternary_weight_only_tern_b200 import synth

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")))


def test_ideal_rate_matches_page():
    b = oracle.bits(4096, 2560, 0)
    assert b["bpw_info"] == math.log2(3)
    assert round(b["bpw_info"], GOLD["ideal_bits_per_trit"]["printed_digits"]) == GOLD["ideal_bits_per_trit"]["value"]


def test_effective_rate_matches_pages_at_printed_second_plane_fraction():
    # the two most salient masks carry a second plane; each printed coverage is rounded to 0.1%
    cov = GOLD["salience_mask_coverage_pct"]
    step = cov["printed_step_pct"] / 2
    two = cov["value"][: cov["two_plane_masks"]]
    lo, hi = sum(two) - step * len(two), sum(two) + step * len(two)
    assert math.isclose(sum(two), GOLD["second_plane_pct"]["value"])
    N = 1_000_000                                      # fine-grained f2
    b_lo = oracle.bits(N, 128, round(N * lo / 100))["bpw_info"]
    b_hi = oracle.bits(N, 128, round(N * hi / 100))["bpw_info"]
    v4 = GOLD["effective_bits_4b"]["value"]
    assert b_lo <= v4 + 5e-4 and v4 - 5e-4 <= b_hi      # 1.641 as printed (+- half a unit in the 3rd digit)
    v8 = GOLD["effective_bits_8b"]["value"]
    assert round(oracle.bits(N, 128, round(N * 0.036))["bpw_info"], 2) == v8


def _serialised_sizes(N, K, r, seed=0):
    rng = np.random.default_rng(seed)
    T1 = synth.draw_trits(rng, (N, K), 0.4)
    T2 = synth.draw_trits(rng, (r, K), 0.4)
    rows = np.sort(rng.choice(N, size=r, replace=False)).astype(np.int32)
    s1 = np.zeros((N, K // 128), np.float16)
    s2 = np.zeros((r, K // 128), np.float16)
    header = 64
    st1, _ = oracle.pack_store(T1)
    st2, _ = oracle.pack_store(T2)
    store = st1.nbytes + st2.nbytes + s1.nbytes + s2.nbytes + oracle.row_bitmap(N, rows).nbytes + header
    ex1, _ = oracle.pack_exec(T1)
    ex2, _ = oracle.pack_exec(T2)
    execb = ex1.nbytes + ex2.nbytes + s1.nbytes + s2.nbytes + oracle.slot_map(N, rows).nbytes + header
    return 8 * store, 8 * execb


@pytest.mark.parametrize("N,K,r", [(16, 128, 0), (24, 256, 5), (13, 384, 13), (8, 1280, 1), (33, 2560, 7)])
def test_bit_totals_equal_serialised_bytes(N, K, r):
    store, execb = _serialised_sizes(N, K, r)
    b = oracle.bits(N, K, r)
    assert b["store_bits"] == store
    assert b["exec_bits"] == execb
    assert b["weights"] == N * K and b["plane_trits"] == (N + r) * K


WORKED = [
    # (N, K, pct) -> info bpw, store bits, exec bits
    ((4096, 2560, 0), 1.584963, 18_092_544, 22_413_824),
    ((9728, 2560, 10), 1.743491, 47_265_856, 58_525_248),
    ((12288, 4096, 15), 1.822681, 99_947_232, 123_389_952),
]


@pytest.mark.parametrize("shape,info,store,execb", WORKED)
def test_worked_values(shape, info, store, execb):
    N, K, pct = shape
    r = synth.residual_count(N, pct)
    b = oracle.bits(N, K, r)
    assert round(b["bpw_info"], 6) == info
    assert b["store_bits"] == store and b["exec_bits"] == execb


def test_targeted_tensor_count():
    t = GOLD["targeted_linear_tensors"]
    assert t["layers"] * len(t["per_layer"]) == t["value"] == synth.N_LAYERS * len(synth.QWEN3_4B)


def test_offset_bits_count_the_serialised_offsets():
    """The offset adds exactly the bits of an fp16 [N, K/128] array to both forms."""
    for (N, K, r) in [(13, 384, 5), (4096, 4096, 614), (1, 128, 0)]:
        a, b = oracle.bits(N, K, r), oracle.bits(N, K, r, offset=True)
        mu_bits = 8 * np.zeros((N, K // 128), np.float16).nbytes
        assert b["store_bits"] - a["store_bits"] == mu_bits
        assert b["exec_bits"] - a["exec_bits"] == mu_bits
        assert b["bpw_info"] == a["bpw_info"]


@pytest.mark.parametrize("N,K,density", [(13, 384, 0.05), (130, 256, 0.036), (64, 128, 0.0)])
def test_elem_bits_count_the_serialised_arrays(N, K, density):
    """exec and store bits of a tensor with an element-level second plane equal the bytes of the
    arrays the oracle serialises: main plane, s1, ecount, ebase (int32), the listed trits, s2e."""
    rng = np.random.default_rng(N + K)
    T1 = synth.draw_trits(rng, (N, K), 0.4)
    mask = rng.random((N, K)) < density
    T2e = np.where(mask, synth.draw_trits(rng, (N, K), 0.4), 0).astype(np.int8)
    c, b, e, _ = oracle.pack_elem(T2e)
    G = K // 128
    elem_bytes = c.nbytes + b.astype(np.int32).nbytes + e.nbytes + np.zeros((N, G), np.float16).nbytes
    s1_bytes = np.zeros((N, G), np.float16).nbytes
    res = oracle.bits_elem(N, K, int(mask.sum()), len(e))
    assert res["exec_bits"] == 8 * (oracle.pack_exec(T1)[0].nbytes + s1_bytes + elem_bytes + 64)
    assert res["store_bits"] == 8 * (oracle.pack_store(T1)[0].nbytes + s1_bytes + elem_bytes + 64)
    assert res["plane_trits"] == N * K + int(mask.sum())
    off = oracle.bits_elem(N, K, int(mask.sum()), len(e), offset=True)
    assert off["exec_bits"] - res["exec_bits"] == 16 * N * G


def test_elem_info_bits_match_pages_at_printed_mask_coverage():
    """The pages' f2 = 3.6 % of weights in the two most salient masks gives the measured
    effective rate (1.641 as printed) when every masked weight counts one more symbol."""
    N, K = 1000, 128 * 1000
    masked = round(N * K * GOLD["second_plane_pct"]["value"] / 100)
    b = oracle.bits_elem(N, K, masked, 0)["bpw_info"]
    assert abs(b - GOLD["effective_bits_4b"]["value"]) <= 5e-4 + math.log2(3) * 0.0005
