"""GPU parity of the multi-token decode kernel (the call takes it for 9 <= M <= 16, and for
4 <= M <= 8 on launches of at least 10 strips per CTA; K a multiple of 512; the other calls run the cluster
kernel and are covered here too): the persistent GEMV whose MMA columns are the tokens. Cases aimed at its structure: one and two 8-token column
blocks and ragged token counts, blocks of 8 and 4 strips (1 and 2 slabs per stage), ranges that
span several segments and weight boundaries, residual rows that fill whole segments, K with an
odd number of 512-wide slabs, offsets, and chains of calls under programmatic dependent launch.

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


def weight(t, mu=None):
    w = api.TernWeight.from_numpy(t.T1, t.s1, t.res_rows, t.T2, t.s2, mu=mu)
    w.static = True
    return w


def run(x, w):
    y = api.linear(torch.from_numpy(np.ascontiguousarray(x)).cuda(), w)
    torch.cuda.synchronize()
    return y.cpu().numpy()


@pytest.mark.parametrize("M", [2, 3, 8, 9, 16])
@pytest.mark.parametrize("K", [512, 2560, 4096, 9728])
@pytest.mark.parametrize("N,pct", [(17, 100), (1000 + 9, 15), (5000, 10)])
def test_shapes_tokens_and_residual_fractions(M, K, N, pct):
    rng = np.random.default_rng(M * 7 + K + N + pct)
    t = synth.draw_tensor(rng, "dm", N, K, M, p_zero=0.4, res_pct=pct)
    check(run(t.x, weight(t)), oracle.linear(t.x, t.T1, t.s1, t.res_rows, t.T2, t.s2))


@pytest.mark.parametrize("M", [2, 3, 4, 5, 7, 8])
@pytest.mark.parametrize("K,pct", [(4096, 15), (12288, 10), (2560, 100)])
def test_one_token_block_on_large_launches(M, K, pct):
    """11 strips per CTA: at M = 4 to 8 one (ragged) 8-token column block in this kernel, x resident
    in shared memory (K = 4096, 2560) or streamed with the stages (K = 12288); at M = 2 and 3 the
    cluster kernel on the same shapes."""
    rng = np.random.default_rng(M * 100 + K + pct)
    N = 148 * 16 * 11 + 5
    t = synth.draw_tensor(rng, "l", N, K, M, p_zero=0.4, res_pct=pct)
    check(run(t.x, weight(t)), oracle.linear(t.x, t.T1, t.s1, t.res_rows, t.T2, t.s2))


@pytest.mark.parametrize("M", [4, 16])
@pytest.mark.parametrize("N,pct", [(50_000, 15), (40_000 + 3, 100)])
def test_many_segments_per_cta(M, N, pct):
    rng = np.random.default_rng(N + M)
    t = synth.draw_tensor(rng, "seg", N, 1024, M, p_zero=0.4, res_pct=pct)
    check(run(t.x, weight(t)), oracle.linear(t.x, t.T1, t.s1, t.res_rows, t.T2, t.s2))


@pytest.mark.parametrize("M", [5, 12])
def test_group_boundaries_inside_cta_ranges(M):
    rng = np.random.default_rng(M)
    x = synth.draw_x(rng, M, 2048)
    ts, ws = [], []
    for N, pct in [(20_000, 15), (16, 0), (7, 100), (3001, 15)]:
        t = synth.draw_tensor(rng, "gb", N, 2048, M, p_zero=0.4, res_pct=pct)
        t = synth.TernTensor("gb", N, 2048, x, t.T1, t.s1, t.res_rows, t.T2, t.s2)
        ts.append(t)
        ws.append(weight(t))
    ys = api.linear_group(torch.from_numpy(x).cuda(), ws)
    torch.cuda.synchronize()
    for y, t in zip(ys, ts):
        check(y.cpu().numpy(), oracle.linear(x, t.T1, t.s1, t.res_rows, t.T2, t.s2))


@pytest.mark.parametrize("M,N,K,r", [(2, 256, 512, 40), (8, 1024 + 5, 4096, 1024 + 5), (16, 130, 12288, 13),
                                     (11, 4000, 2560, 600), (5, 148 * 16 * 11, 4096, 3000)])
def test_exact_case_bit_exact(M, N, K, r):
    rng = np.random.default_rng(M + N * 3 + K + r)
    t = synth.draw_exact_tensor(rng, N, K, M, r)
    for mu in (None, synth.draw_exact_offsets(rng, N, K)):
        y_ref = oracle.round_fp16(oracle.linear(t.x, t.T1, t.s1, t.res_rows, t.T2, t.s2, mu=mu))
        assert np.array_equal(run(t.x, weight(t, mu)).view(np.uint16), y_ref.view(np.uint16))


@pytest.mark.parametrize("M", [3, 16])
def test_zero_plane_is_exactly_zero_and_offsets(M):
    rng = np.random.default_rng(80 + M)
    N, K = 300, 4096
    x = synth.draw_x(rng, M, K)
    s1 = synth.draw_scales(rng, N, K, 0.005, 0.02)
    none = (np.zeros(0, np.int32), np.zeros((0, K), np.int8), np.zeros((0, K // 128), np.float16))
    z = synth.TernTensor("z", N, K, x, np.zeros((N, K), np.int8), s1, *none)
    assert (run(x, weight(z)) == 0).all()
    t = synth.draw_tensor(rng, "m", N, K, M, p_zero=0.4, res_pct=15)
    mu = synth.draw_offsets(rng, N, K)
    check(run(t.x, weight(t, mu)), oracle.linear(t.x, t.T1, t.s1, t.res_rows, t.T2, t.s2, mu=mu))


def test_non_finite_activation_makes_only_its_token_non_finite():
    rng = np.random.default_rng(41)
    t = synth.draw_tensor(rng, "nan", 200, 1024, 6, p_zero=0.4, res_pct=10)
    x = t.x.copy()
    x[2, 700] = np.inf
    y = run(x, weight(t))
    assert not np.isfinite(y[2]).any()
    keep = [0, 1, 3, 4, 5]
    ref = oracle.linear(t.x[keep], t.T1, t.s1, t.res_rows, t.T2, t.s2)
    check(y[keep], ref)


def test_deterministic_across_calls():
    t = next(synth.draw_workload(synth.WORKLOADS[4], only=["gate"]))
    x = synth.draw_x(np.random.default_rng(5), 16, t.K)
    w = weight(t)
    a, b = run(x, w), run(x, w)
    assert np.array_equal(a.view(np.uint16), b.view(np.uint16))


def test_chain_of_overlapping_calls_reads_each_input_after_it_is_written():
    rng = np.random.default_rng(13)
    N = K = 2048
    M = 7
    ts = [synth.draw_tensor(rng, f"c{i}", N, K, M, p_zero=0.4, res_pct=15) for i in range(5)]
    ws = [weight(t) for t in ts]
    h = torch.from_numpy(ts[0].x).cuda()
    for w in ws:
        h = api.linear(h, w)
    torch.cuda.synchronize()
    ref = ts[0].x.astype(np.float64)
    for t in ts:
        ref = oracle.round_fp16(oracle.linear(ref.astype(np.float16), t.T1, t.s1, t.res_rows, t.T2, t.s2))
    check(h.cpu().numpy(), ref.astype(np.float64), tol=5e-3)
