"""GPU parity of the one-token decode kernel (M = 1, K a multiple of 512): the persistent,
warp-specialised GEMV that streams 16-row strips. Cases aimed at its structure: ranges of strips
that span several 256-row segments and weight boundaries, residual rows that fill whole segments,
K split over several stages, uneven splits of the groups over the consumer warps, ragged N, and
chains of calls that overlap under programmatic dependent launch.

Bar: max|y - y_ref| / max|y_ref| <= 2e-3 against the float64 oracle, and bit-exact equality with
the oracle's single fp16 rounding on inputs where fp32 accumulation is exact.
"""

import numpy as np
import pytest
import torch

import oracle
from ternary_weight_only_tern_b200 import api, synth

pytestmark = pytest.mark.gpu
TOL = 2e-3


def check(y, y_ref, tol=TOL):
    assert np.isfinite(y).all()
    err = oracle.rel_err(y.astype(np.float64), y_ref)
    assert err <= tol, f"rel err {err:.3e}"


def weight(t, mu=None, static=False):
    w = api.TernWeight.from_numpy(t.T1, t.s1, t.res_rows, t.T2, t.s2, mu=mu)
    w.static = static
    return w


def one(x, w):
    y = api.linear(torch.from_numpy(np.ascontiguousarray(x[:1])).cuda(), w)
    torch.cuda.synchronize()
    return y.cpu().numpy()


# K = 512 .. 12288: one group per warp up to 4, several stages per strip, W = 8 or 10 warps
@pytest.mark.parametrize("K", [512, 1024, 2560, 4608, 9728, 12288])
@pytest.mark.parametrize("N,pct", [(16, 0), (17, 100), (1000 + 9, 15), (4096, 10)])
def test_shapes_and_residual_fractions(K, N, pct):
    rng = np.random.default_rng(K + N + pct)
    t = synth.draw_tensor(rng, "d1", N, K, 1, p_zero=0.4, res_pct=pct)
    check(one(t.x, weight(t)), oracle.linear(t.x, t.T1, t.s1, t.res_rows, t.T2, t.s2))


@pytest.mark.parametrize("N,pct", [(50_000, 15), (50_000 + 3, 100), (2 * 148 * 16 + 5, 0)])
def test_many_segments_per_cta(N, pct):
    """More than 256 rows per CTA: the range is cut into several segments, each with its own
    residual slots (all rows residual: 16 residual strips per segment)."""
    rng = np.random.default_rng(N)
    t = synth.draw_tensor(rng, "seg", N, 512, 1, p_zero=0.4, res_pct=pct)
    check(one(t.x, weight(t)), oracle.linear(t.x, t.T1, t.s1, t.res_rows, t.T2, t.s2))


@pytest.mark.parametrize("shapes", [[(40_000, 15), (16, 0), (7, 100), (3001, 15)], [(1, 100), (1, 0)]])
def test_group_boundaries_inside_cta_ranges(shapes):
    rng = np.random.default_rng(len(shapes))
    x = synth.draw_x(rng, 1, 1024)
    ts, ws = [], []
    for N, pct in shapes:
        t = synth.draw_tensor(rng, "gb", N, 1024, 1, p_zero=0.4, res_pct=pct)
        t = synth.TernTensor("gb", N, 1024, x, t.T1, t.s1, t.res_rows, t.T2, t.s2)
        ts.append(t)
        ws.append(weight(t))
    ys = api.linear_group(torch.from_numpy(x).cuda(), ws)
    torch.cuda.synchronize()
    for y, t in zip(ys, ts):
        check(y.cpu().numpy(), oracle.linear(x, t.T1, t.s1, t.res_rows, t.T2, t.s2))


@pytest.mark.parametrize("N,K,r", [(256, 512, 40), (1024 + 5, 4096, 1024 + 5), (130, 12288, 13), (4000, 2560, 600)])
def test_exact_case_bit_exact(N, K, r):
    rng = np.random.default_rng(N * 3 + K + r)
    t = synth.draw_exact_tensor(rng, N, K, 1, r)
    y_ref = oracle.round_fp16(oracle.linear(t.x, t.T1, t.s1, t.res_rows, t.T2, t.s2))
    for mu in (None, synth.draw_exact_offsets(rng, N, K)):
        if mu is not None:
            y_ref = oracle.round_fp16(oracle.linear(t.x, t.T1, t.s1, t.res_rows, t.T2, t.s2, mu=mu))
        assert np.array_equal(one(t.x, weight(t, mu)).view(np.uint16), y_ref.view(np.uint16))


def test_zero_plane_is_exactly_zero_and_all_ones_is_the_group_sum():
    rng = np.random.default_rng(8)
    N, K = 300, 4096
    x = synth.draw_x(rng, 1, K)
    s1 = synth.draw_scales(rng, N, K, 0.005, 0.02)
    none = (np.zeros(0, np.int32), np.zeros((0, K), np.int8), np.zeros((0, K // 128), np.float16))
    z = synth.TernTensor("z", N, K, x, np.zeros((N, K), np.int8), s1, *none)
    assert (one(x, weight(z)) == 0).all()
    p = synth.TernTensor("p", N, K, x, np.ones((N, K), np.int8), s1, *none)
    check(one(x, weight(p)), oracle.linear(x, p.T1, s1, *none))


def test_offsets_on_some_weights_of_a_group():
    rng = np.random.default_rng(21)
    x = synth.draw_x(rng, 1, 2560)
    ts, mus, ws = [], [], []
    for N, with_mu in ((512, True), (130, False), (1000 + 7, True)):
        t = synth.draw_tensor(rng, "m", N, 2560, 1, p_zero=0.4, res_pct=15)
        t = synth.TernTensor("m", N, 2560, x, t.T1, t.s1, t.res_rows, t.T2, t.s2)
        mu = synth.draw_offsets(rng, N, 2560) if with_mu else None
        ts.append(t)
        mus.append(mu)
        ws.append(weight(t, mu))
    ys = api.linear_group(torch.from_numpy(x).cuda(), ws)
    torch.cuda.synchronize()
    for y, t, mu in zip(ys, ts, mus):
        check(y.cpu().numpy(), oracle.linear(x, t.T1, t.s1, t.res_rows, t.T2, t.s2, mu=mu))


def test_non_finite_activation_makes_the_token_non_finite():
    rng = np.random.default_rng(4)
    t = synth.draw_tensor(rng, "nan", 200, 1024, 1, p_zero=0.4, res_pct=10)
    x = t.x.copy()
    x[0, 700] = np.inf
    y = one(x, weight(t))
    assert not np.isfinite(y).any()


def test_deterministic_across_calls_and_static_flag():
    t = next(synth.draw_workload(synth.WORKLOADS[4], only=["gate"]))
    a, b = one(t.x, weight(t)), one(t.x, weight(t, static=True))
    c = one(t.x, weight(t, static=True))
    assert np.array_equal(a.view(np.uint16), b.view(np.uint16))
    assert np.array_equal(b.view(np.uint16), c.view(np.uint16))


def test_chain_of_overlapping_calls_reads_each_input_after_it_is_written():
    """Each call's x is the previous call's y; the calls overlap under programmatic dependent
    launch (static weights start streaming early), and every call must still read its input only
    once it is complete."""
    rng = np.random.default_rng(12)
    N = K = 2048
    ts = [synth.draw_tensor(rng, f"c{i}", N, K, 1, p_zero=0.4, res_pct=15) for i in range(6)]
    ws = [weight(t, static=True) for t in ts]
    h = torch.from_numpy(ts[0].x).cuda()
    for w in ws:
        h = api.linear(h, w)
    torch.cuda.synchronize()
    ref = ts[0].x.astype(np.float64)
    for t in ts:
        ref = oracle.round_fp16(oracle.linear(ref.astype(np.float16), t.T1, t.s1, t.res_rows, t.T2, t.s2))
    check(h.cpu().numpy(), ref.astype(np.float64), tol=5e-3)


def test_graph_replay_with_new_inputs():
    t = next(synth.draw_workload(synth.WORKLOADS[4], only=["o"]))
    w = weight(t, static=True)
    x = torch.zeros((1, t.K), dtype=torch.float16, device="cuda")
    y = torch.empty((1, t.N), dtype=torch.float16, device="cuda")
    api.linear(x, w, out=y)            # configure outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        api.linear(x, w, out=y)
    rng = np.random.default_rng(3)
    for _ in range(3):
        xn = synth.draw_x(rng, 1, t.K)
        x.copy_(torch.from_numpy(xn))
        g.replay()
        torch.cuda.synchronize()
        check(y.cpu().numpy(), oracle.linear(xn, t.T1, t.s1, t.res_rows, t.T2, t.s2))


@pytest.mark.parametrize("M", [1, 5, 16])
@pytest.mark.parametrize("pct", [15, 100])
def test_balanced_split_gives_the_same_bits(M, pct):
    """A launch whose CTAs' strip ranges are balanced by the weights' residual rows per strip
    (the host hint) computes every row in the same order as the even split: the outputs are
    bit-identical, and within the bar against the oracle. Gate-and-up-like group of two weights
    (11 strips per CTA), rows with residual rows bunched at one end."""
    import dataclasses

    rng = np.random.default_rng(300 + M + pct)
    K = 2048
    x = synth.draw_x(rng, M, K)
    ts, hinted, plain = [], [], []
    for i, N in enumerate((148 * 16 * 6, 148 * 16 * 5 + 7)):
        t = synth.draw_tensor(rng, "bal", N, K, M, p_zero=0.4, res_pct=pct)
        if pct < 100:   # residual rows bunched into the first third of the rows
            r = t.res_rows.size
            rows = np.sort(rng.choice(N // 3, size=min(r, N // 3), replace=False)).astype(np.int32)
            T2 = synth.draw_trits(rng, (rows.size, K), p_zero=0.4)
            s2 = synth.draw_scales(rng, rows.size, K, 0.001, 0.005)
            t = synth.TernTensor("bal", N, K, x, t.T1, t.s1, rows, T2, s2)
        else:
            t = synth.TernTensor("bal", N, K, x, t.T1, t.s1, t.res_rows, t.T2, t.s2)
        ts.append(t)
        w = weight(t)
        assert w.res_hint is not None and int(w.res_hint.sum()) == t.res_rows.size
        hinted.append(w)
        plain.append(dataclasses.replace(w, res_hint=None))
    xt = torch.from_numpy(x).cuda()
    ya = api.linear_group(xt, hinted)
    yb = api.linear_group(xt, plain)
    torch.cuda.synchronize()
    for a, b, t in zip(ya, yb, ts):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
        check(a.cpu().numpy(), oracle.linear(x, t.T1, t.s1, t.res_rows, t.T2, t.s2))
