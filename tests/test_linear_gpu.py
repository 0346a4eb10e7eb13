"""GPU parity of tern_linear against the float64 oracle.

Bar: max|y - y_ref| / max|y_ref| <= 2e-3 with no NaN/Inf on seeded synthetic inputs, and
bit-exact equality with the oracle's single fp16 rounding on inputs where fp32 accumulation is
exact. Full-size shapes of all five workloads run in the launch configuration the bench times;
where the oracle would be slow (the 36-layer stack, M = 2048) it computes sampled output
columns for every token.
"""

import numpy as np
import pytest
import torch

import oracle
from ternary_weight_only_tern_b200 import api, synth

pytestmark = pytest.mark.gpu
TOL = 2e-3


def run(t: synth.TernTensor, M: int, weight=None):
    w = weight or api.TernWeight.from_numpy(t.T1, t.s1, t.res_rows, t.T2, t.s2)
    x = torch.from_numpy(np.ascontiguousarray(t.x[:M])).cuda()
    y = api.linear(x, w)
    torch.cuda.synchronize()
    return y.cpu().numpy(), w


def check(y, y_ref, tol=TOL):
    assert np.isfinite(y).all()
    err = oracle.rel_err(y.astype(np.float64), y_ref)
    assert err <= tol, f"rel err {err:.3e}"
    return err


def test_config1_single_gemv():
    t = next(synth.draw_workload(synth.WORKLOADS[1]))
    y, _ = run(t, 1)
    check(y, oracle.linear(t.x[:1], t.T1, t.s1, t.res_rows, t.T2, t.s2))


@pytest.mark.parametrize("name", list(synth.QWEN3_4B))
def test_config2_4b_layer(name):
    t = next(synth.draw_workload(synth.WORKLOADS[2], only=[name]))
    y, _ = run(t, 1)
    check(y, oracle.linear(t.x[:1], t.T1, t.s1, t.res_rows, t.T2, t.s2))


@pytest.mark.parametrize("name", list(synth.QWEN3_8B))
def test_config4_8b_projections_all_M(name):
    t = next(synth.draw_workload(synth.WORKLOADS[4], only=[name]))
    y_ref = oracle.linear(t.x, t.T1, t.s1, t.res_rows, t.T2, t.s2)       # 16 tokens
    w = None
    for M in synth.WORKLOADS[4].Ms:
        y, w = run(t, M, w)
        check(y, y_ref[:M])


@pytest.mark.parametrize("layer", range(36))
def test_config3_4b_stack_sampled(layer):
    """Every layer of the 36-layer Qwen3-4B stack (252 tensors), each projection at M = 1, 4 and 16,
    on sampled output columns (including residual rows) against the column-restricted oracle."""
    rng = np.random.default_rng(layer)
    for t in synth.draw_workload(synth.WORKLOADS[3], layers=[layer]):
        cols = np.unique(np.concatenate([rng.choice(t.N, 48, replace=False), t.res_rows[:16]]))
        y_ref = oracle.linear(t.x, t.T1, t.s1, t.res_rows, t.T2, t.s2, cols=cols)
        w = None
        for M in synth.WORKLOADS[3].Ms:
            y, w = run(t, M, w)
            check(y[:, cols], y_ref[:M])


@pytest.mark.parametrize("name", ["gate", "up", "down"])
def test_config5_prefill_sampled(name):
    t = next(synth.draw_workload(synth.WORKLOADS[5], only=[name]))
    rng = np.random.default_rng(5)
    cols = np.unique(np.concatenate([rng.choice(t.N, 40, replace=False), t.res_rows[:24]]))
    y_ref = oracle.linear(t.x, t.T1, t.s1, t.res_rows, t.T2, t.s2, cols=cols)
    y, _ = run(t, 2048)
    check(y[:, cols], y_ref)


@pytest.mark.parametrize("M", [1, 2, 3, 5, 8, 9, 15, 16, 17, 100, 511, 513])
def test_odd_M(M):
    rng = np.random.default_rng(100 + M)
    t = synth.draw_tensor(rng, "odd", 320, 1152, M, p_zero=0.4, res_pct=10)
    y, _ = run(t, M)
    check(y, oracle.linear(t.x, t.T1, t.s1, t.res_rows, t.T2, t.s2))


@pytest.mark.parametrize("N,K,r", [(100, 128, 7), (1, 128, 1), (1000 + 7, 384, 0), (77, 12288, 77), (64, 256, 64),
                                   (4096 + 48, 2560, 300)])
def test_ragged_and_degenerate_shapes(N, K, r):
    rng = np.random.default_rng(N + K + r)
    t = synth.draw_tensor(rng, "rag", N, K, 16, p_zero=0.4, res_pct=0)
    rr = np.sort(rng.choice(N, r, replace=False)).astype(np.int32)
    T2 = synth.draw_trits(rng, (r, K), 0.4)
    s2 = synth.draw_scales(rng, r, K, 0.001, 0.005)
    t = synth.TernTensor("rag", N, K, t.x, t.T1, t.s1, rr, T2, s2)
    y_ref = oracle.linear(t.x, t.T1, t.s1, rr, T2, s2)
    w = None
    for M in (1, 7, 16):
        y, w = run(t, M, w)
        check(y, y_ref[:M])


@pytest.mark.parametrize("M", [1, 4, 8, 16, 24, 300])
@pytest.mark.parametrize("N,K,r", [(256, 512, 40), (1024, 4096, 154), (130, 12288, 13)])
def test_exact_case_bit_exact(M, N, K, r):
    rng = np.random.default_rng(M * 31 + N + K)
    t = synth.draw_exact_tensor(rng, N, K, M, r)
    y, _ = run(t, M)
    y_ref = oracle.round_fp16(oracle.linear(t.x, t.T1, t.s1, t.res_rows, t.T2, t.s2))
    assert np.array_equal(y.view(np.uint16), y_ref.view(np.uint16))


def test_special_cases():
    rng = np.random.default_rng(77)
    N, K, M = 192, 512, 16
    x = synth.draw_x(rng, M, K)
    s1 = synth.draw_scales(rng, N, K, 0.005, 0.02)
    none = (np.zeros(0, np.int32), np.zeros((0, K), np.int8), np.zeros((0, K // 128), np.float16))
    # zero plane -> exactly zero
    t = synth.TernTensor("z", N, K, x, np.zeros((N, K), np.int8), s1, *none)
    y, _ = run(t, M)
    assert (y == 0).all()
    # all +1: s times group sums
    t = synth.TernTensor("p", N, K, x, np.ones((N, K), np.int8), s1, *none)
    y, _ = run(t, M)
    check(y, oracle.linear(x, t.T1, s1, *none))
    # r = N with T2 = T1, s2 = s1 doubles the r = 0 result
    T1 = synth.draw_trits(rng, (N, K), 0.4)
    y1, _ = run(synth.TernTensor("a", N, K, x, T1, s1, *none), M)
    y2, _ = run(synth.TernTensor("b", N, K, x, T1, s1, np.arange(N, dtype=np.int32), T1, s1), M)
    check(y2, 2 * y1.astype(np.float64), tol=1e-3)


def test_out_shape_is_checked():
    t = next(synth.draw_workload(synth.WORKLOADS[1]))
    w = api.TernWeight.from_numpy(t.T1, t.s1, t.res_rows, t.T2, t.s2)
    x = torch.from_numpy(t.x).cuda()
    with pytest.raises(ValueError):
        api.linear(x, w, out=torch.empty((2, t.N), dtype=torch.float16, device="cuda"))


def test_deterministic_and_m0():
    t = next(synth.draw_workload(synth.WORKLOADS[4], only=["q"]))
    y1, w = run(t, 16)
    y2, _ = run(t, 16, w)
    assert np.array_equal(y1.view(np.uint16), y2.view(np.uint16))
    x = torch.empty((0, t.K), dtype=torch.float16, device="cuda")
    assert api.linear(x, w).shape == (0, t.N)


@pytest.mark.parametrize("M", [3, 40])
def test_non_finite_activations_propagate(M):
    """A token with an inf or NaN activation gets non-finite outputs (the oracle's IEEE sums give
    +-inf or NaN there); the other tokens stay finite and within tolerance."""
    rng = np.random.default_rng(3)
    t = synth.draw_tensor(rng, "nan", 64, 256, M, p_zero=0.4, res_pct=10)
    x = t.x.copy()
    x[0, 5] = np.inf
    x[1, 7] = np.nan
    t = synth.TernTensor("n", 64, 256, x, t.T1, t.s1, t.res_rows, t.T2, t.s2)
    y, _ = run(t, M)
    with np.errstate(invalid="ignore"):
        y_ref = oracle.linear(x, t.T1, t.s1, t.res_rows, t.T2, t.s2)
    assert not np.isfinite(y_ref[:2]).any()
    assert not np.isfinite(y[:2]).any()
    check(y[2:], y_ref[2:])


def test_workspace_and_output_untouched_outside_bounds():
    t = next(synth.draw_workload(synth.WORKLOADS[4], only=["k"]))
    w = api.TernWeight.from_numpy(t.T1, t.s1, t.res_rows, t.T2, t.s2)
    M = 16
    assert t.x.shape[0] == M
    need = api.workspace_bytes(w, M)
    ws = torch.full((need + 4096,), 0xA5, dtype=torch.uint8, device="cuda")
    yb = torch.full((M * t.N + 4096,), 7.0, dtype=torch.float16, device="cuda")
    x = torch.from_numpy(t.x[:M]).cuda()
    api.linear(x, w, out=yb[: M * t.N].view(M, t.N), workspace=ws)
    torch.cuda.synchronize()
    assert (ws[need:] == 0xA5).all() and (yb[M * t.N:] == 7.0).all()
    check(yb[: M * t.N].view(M, t.N).cpu().numpy(), oracle.linear(t.x[:M], t.T1, t.s1, t.res_rows, t.T2, t.s2))


@pytest.mark.parametrize("M", [1, 16, 64])
def test_static_weight_flag_gives_the_same_bits(M):
    t = next(synth.draw_workload(synth.WORKLOADS[4], only=["o"]))
    rng = np.random.default_rng(M)
    x = torch.from_numpy(synth.draw_x(rng, M, t.K)).cuda()
    w = api.TernWeight.from_numpy(t.T1, t.s1, t.res_rows, t.T2, t.s2)
    ws = api.TernWeight.from_numpy(t.T1, t.s1, t.res_rows, t.T2, t.s2)
    ws.static = True
    y1, y2 = api.linear(x, w), api.linear(x, ws)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_back_to_back_calls_on_one_stream_see_their_inputs():
    """Consecutive calls overlap under programmatic dependent launch; each must read the x that
    the previous call wrote (a two-layer chain), and the result must match the oracle's chain."""
    rng = np.random.default_rng(11)
    N, K = 1024, 1024
    ts = [synth.draw_tensor(rng, f"c{i}", N, K, 4, p_zero=0.4, res_pct=15) for i in range(3)]
    ws = [api.TernWeight.from_numpy(t.T1, t.s1, t.res_rows, t.T2, t.s2) for t in ts]
    for w in ws:
        w.static = True
    x = torch.from_numpy(ts[0].x).cuda()
    h = x
    for w in ws:
        h = api.linear(h, w)
    torch.cuda.synchronize()
    ref = ts[0].x.astype(np.float64)
    for t in ts:
        ref = oracle.round_fp16(oracle.linear(ref.astype(np.float16), t.T1, t.s1, t.res_rows, t.T2, t.s2))
    check(h.cpu().numpy(), ref.astype(np.float64), tol=5e-3)


def test_device_status_is_clean_after_the_suite():
    from ternary_weight_only_tern_b200 import _lib
    assert _lib.load().tern_device_status(api._stream()) == 0


@pytest.mark.parametrize("M", [1, 5, 16, 40])
def test_prefetch_of_the_next_weight_changes_nothing(M):
    """tern_linear_with_prefetch gives the same bits as tern_linear; the next weight (here of a
    different shape, with residual rows) is only a cache hint."""
    a = next(synth.draw_workload(synth.WORKLOADS[4], only=["q"]))
    b = next(synth.draw_workload(synth.WORKLOADS[4], only=["down"]))
    wa = api.TernWeight.from_numpy(a.T1, a.s1, a.res_rows, a.T2, a.s2)
    wb = api.TernWeight.from_numpy(b.T1, b.s1, b.res_rows, b.T2, b.s2)
    x = torch.from_numpy(np.ascontiguousarray(np.resize(a.x, (M, a.K)))).cuda()
    y1 = api.linear(x, wa)
    y2 = api.linear(x, wa, prefetch=wb)
    y3 = api.linear(x, wa, prefetch=wa)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    assert torch.equal(y1.view(torch.int16), y3.view(torch.int16))


# ---------------------------------------------------------------- per-group offset mu
def run_mu(t: synth.TernTensor, mu: np.ndarray, M: int, weight=None):
    w = weight or api.TernWeight.from_numpy(t.T1, t.s1, t.res_rows, t.T2, t.s2, mu=mu)
    return run(t, M, w)


@pytest.mark.parametrize("M", [1, 2, 4, 8, 9, 16, 17, 300])
@pytest.mark.parametrize("N,K,pct", [(320, 1152, 10), (1000 + 7, 12288, 15), (64, 128, 100)])
def test_offset_parity(M, N, K, pct):
    rng = np.random.default_rng(7 * M + N + K)
    t = synth.draw_tensor(rng, "mu", N, K, M, p_zero=0.4, res_pct=pct)
    mu = synth.draw_offsets(rng, N, K)
    y, _ = run_mu(t, mu, M)
    check(y, oracle.linear(t.x, t.T1, t.s1, t.res_rows, t.T2, t.s2, mu=mu))


@pytest.mark.parametrize("M", [1, 4, 16, 24, 300])
@pytest.mark.parametrize("N,K,r", [(256, 512, 40), (130, 12288, 13)])
def test_offset_exact_case_bit_exact(M, N, K, r):
    rng = np.random.default_rng(M * 17 + N + K)
    t = synth.draw_exact_tensor(rng, N, K, M, r)
    mu = synth.draw_exact_offsets(rng, N, K)
    y, _ = run_mu(t, mu, M)
    y_ref = oracle.round_fp16(oracle.linear(t.x, t.T1, t.s1, t.res_rows, t.T2, t.s2, mu=mu))
    assert np.array_equal(y.view(np.uint16), y_ref.view(np.uint16))


@pytest.mark.parametrize("M", [1, 5, 16, 40])
def test_zero_offset_gives_the_bits_of_no_offset(M):
    rng = np.random.default_rng(300 + M)
    t = synth.draw_tensor(rng, "mu0", 512, 2560, M, p_zero=0.4, res_pct=10)
    y0, _ = run(t, M)
    y1, _ = run_mu(t, np.zeros((t.N, t.K // 128), np.float16), M)
    assert np.array_equal(y0.view(np.uint16), y1.view(np.uint16))


@pytest.mark.parametrize("M", [1, 16, 2048])
def test_offset_8b_gate_full_size(M):
    t = next(synth.draw_workload(synth.WORKLOADS[5], only=["gate"]))
    rng = np.random.default_rng(11)
    mu = synth.draw_offsets(rng, t.N, t.K)
    cols = np.unique(np.concatenate([rng.choice(t.N, 40, replace=False), t.res_rows[:24]]))
    y_ref = oracle.linear(t.x[:M], t.T1, t.s1, t.res_rows, t.T2, t.s2, cols=cols, mu=mu)
    y, _ = run_mu(t, mu, M)
    check(y[:, cols], y_ref)


# ---------------------------------------------------------------- weights sharing one input
def _group_tensors(rng, shapes, M, res_pct=10):
    x = synth.draw_x(rng, M, shapes[0][1])
    out = []
    for N, K in shapes:
        t = synth.draw_tensor(rng, "g", N, K, 1, p_zero=0.4, res_pct=res_pct)
        out.append(synth.TernTensor("g", N, K, x, t.T1, t.s1, t.res_rows, t.T2, t.s2))
    return x, out


@pytest.mark.parametrize("M", [1, 3, 8, 16, 17, 40])
@pytest.mark.parametrize("which", ["qkv", "gateup"])
def test_group_matches_oracle(M, which):
    names = ["q", "k", "v"] if which == "qkv" else ["gate", "up"]
    rng = np.random.default_rng(M + len(which))
    x, ts = _group_tensors(rng, [synth.QWEN3_8B[n] for n in names], M, res_pct=15)
    ws = [api.TernWeight.from_numpy(t.T1, t.s1, t.res_rows, t.T2, t.s2) for t in ts]
    ys = api.linear_group(torch.from_numpy(x).cuda(), ws)
    torch.cuda.synchronize()
    for y, t in zip(ys, ts):
        check(y.cpu().numpy(), oracle.linear(x, t.T1, t.s1, t.res_rows, t.T2, t.s2))


@pytest.mark.parametrize("M", [1, 4, 16, 24])
def test_group_exact_case_bit_exact(M):
    rng = np.random.default_rng(900 + M)
    ts = [synth.draw_exact_tensor(rng, N, 1536, M, r) for N, r in [(300, 17), (64, 0), (1000 + 7, 100), (130, 130)]]
    x = ts[0].x
    ws = [api.TernWeight.from_numpy(t.T1, t.s1, t.res_rows, t.T2, t.s2) for t in ts]
    ys = api.linear_group(torch.from_numpy(x).cuda(), ws)
    torch.cuda.synchronize()
    for y, t in zip(ys, ts):
        y_ref = oracle.round_fp16(oracle.linear(x, t.T1, t.s1, t.res_rows, t.T2, t.s2))
        assert np.array_equal(y.cpu().numpy().view(np.uint16), y_ref.view(np.uint16))


@pytest.mark.parametrize("M", [1, 5, 16])
def test_group_of_one_is_tern_linear_and_prefetch_changes_nothing(M):
    rng = np.random.default_rng(70 + M)
    t = synth.draw_tensor(rng, "g1", 1000 + 7, 2560, M, p_zero=0.4, res_pct=10)
    w = api.TernWeight.from_numpy(t.T1, t.s1, t.res_rows, t.T2, t.s2)
    x = torch.from_numpy(t.x).cuda()
    y0 = api.linear(x, w)
    (y1,) = api.linear_group(x, [w])
    (y2,) = api.linear_group(x, [w], prefetch=[w, w, w])
    torch.cuda.synchronize()
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))
    assert torch.equal(y0.view(torch.int16), y2.view(torch.int16))


@pytest.mark.parametrize("M", [1, 9, 300])
def test_group_with_offsets_and_element_planes(M):
    rng = np.random.default_rng(55 + M)
    x = synth.draw_x(rng, M, 2560)
    refs, ws = [], []
    for N in (512, 130, 1000 + 7):
        T1 = synth.draw_trits(rng, (N, 2560), 0.4)
        s1 = synth.draw_scales(rng, N, 2560, 0.005, 0.02)
        T2e, s2e, _ = synth.draw_elem_plane(rng, N, 2560)
        mu = synth.draw_offsets(rng, N, 2560)
        none = (np.zeros(0, np.int32), np.zeros((0, 2560), np.int8), np.zeros((0, 20), np.float16))
        ws.append(api.TernWeight.from_numpy(T1, s1, *none, mu=mu, T2e=T2e, s2e=s2e))
        refs.append(oracle.linear(x, T1, s1, *none, mu=mu, elem=(T2e, s2e)))
    ys = api.linear_group(torch.from_numpy(x).cuda(), ws)
    torch.cuda.synchronize()
    for y, y_ref in zip(ys, refs):
        check(y.cpu().numpy(), y_ref)
