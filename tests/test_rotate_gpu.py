"""GPU parity of tern_rotate (the activation-side block rotation) against the oracle.

max|y - y_ref| / max|y_ref| <= 2e-3 on seeded inputs at M from 1 to 2048 (sampled tokens at
2048) and K from 128 to 12288; bit-exact where fp32 accumulation is exact (integer x, dyadic R);
identity blocks return x; and a rotation followed by tern_linear on the rotated weight matches the
oracle's product with the original weight.
"""

import numpy as np
import pytest
import torch

import oracle
from ternary_weight_only_tern_b200 import api, synth

pytestmark = pytest.mark.gpu
TOL = 2e-3


def _orthogonal(rng, G):
    out = np.empty((G, 128, 128))
    for g in range(G):
        q, r = np.linalg.qr(rng.standard_normal((128, 128)))
        out[g] = q * np.sign(np.diag(r))
    return out


def _rot(x, R):
    y = api.rotate(torch.from_numpy(np.ascontiguousarray(x)).cuda(), torch.from_numpy(R).cuda())
    torch.cuda.synchronize()
    return y.cpu().numpy()


@pytest.mark.parametrize("M", [1, 2, 15, 16, 17, 64, 65, 300])
@pytest.mark.parametrize("K", [128, 384, 4096, 12288])
def test_rotate_matches_oracle(M, K):
    rng = np.random.default_rng(M * 7 + K)
    x = synth.draw_x(rng, M, K)
    R = _orthogonal(rng, K // 128).astype(np.float16)
    y = _rot(x, R)
    y_ref = oracle.rotate(x, R)
    assert np.isfinite(y).all()
    assert oracle.rel_err(y.astype(np.float64), y_ref) <= TOL


def test_rotate_m2048_sampled_tokens():
    rng = np.random.default_rng(2048)
    x = synth.draw_x(rng, 2048, 4096)
    R = _orthogonal(rng, 32).astype(np.float16)
    y = _rot(x, R)
    rows = rng.choice(2048, 64, replace=False)
    assert oracle.rel_err(y[rows].astype(np.float64), oracle.rotate(x[rows], R)) <= TOL


@pytest.mark.parametrize("M", [1, 5, 64, 130])
def test_rotate_exact_case_bit_exact(M):
    rng = np.random.default_rng(M)
    x = rng.integers(-4, 5, size=(M, 512)).astype(np.float16)
    R = (rng.integers(-8, 9, size=(4, 128, 128)) / 16).astype(np.float16)
    y = _rot(x, R)
    y_ref = oracle.round_fp16(oracle.rotate(x, R))
    assert np.array_equal(y.view(np.uint16), y_ref.view(np.uint16))


def test_rotate_by_identity_returns_x():
    rng = np.random.default_rng(3)
    x = synth.draw_x(rng, 33, 1024)
    y = _rot(x, np.stack([np.eye(128, dtype=np.float16)] * 8))
    assert np.array_equal(y.view(np.uint16), x.view(np.uint16))


@pytest.mark.parametrize("M", [1, 16, 40])
def test_rotation_then_linear_on_the_rotated_weight(M):
    """x' = tern_rotate(x, R), y = tern_linear(x', W') where W' is a ternary weight given in the
    rotated basis; the oracle computes the same chain from x in float64 (the rotation rounded to
    fp16 once, as the kernel's output is)."""
    rng = np.random.default_rng(60 + M)
    t = synth.draw_tensor(rng, "rot", 1000 + 7, 2560, M, p_zero=0.4, res_pct=10)
    R = _orthogonal(rng, 20).astype(np.float16)
    w = api.TernWeight.from_numpy(t.T1, t.s1, t.res_rows, t.T2, t.s2)
    xd = torch.from_numpy(t.x).cuda()
    xrd = api.rotate(xd, torch.from_numpy(R).cuda())
    y = api.linear(xrd, w)
    torch.cuda.synchronize()
    x_rot_ref = oracle.round_fp16(oracle.rotate(t.x, R))
    y_ref = oracle.linear(x_rot_ref, t.T1, t.s1, t.res_rows, t.T2, t.s2)
    assert oracle.rel_err(y.cpu().numpy().astype(np.float64), y_ref) <= TOL


@pytest.mark.parametrize("M", [1, 4, 130])
def test_rotation_and_groups_chained_in_a_cuda_graph(M):
    """rotate -> linear_group -> rotate -> linear, captured once in a CUDA graph and replayed with new
    inputs: every launch (several with programmatic dependent launch) reads what the one before
    it wrote, and each replay matches the oracle's chain."""
    rng = np.random.default_rng(90 + M)
    K = 1024
    R1 = _orthogonal(rng, K // 128).astype(np.float16)
    ts = [synth.draw_tensor(rng, f"g{i}", 1024, K, M, p_zero=0.4, res_pct=10) for i in range(2)]
    ws = [api.TernWeight.from_numpy(t.T1, t.s1, t.res_rows, t.T2, t.s2) for t in ts]
    for w in ws:
        w.static = True
    R1d = torch.from_numpy(R1).cuda()
    x = torch.zeros((M, K), dtype=torch.float16, device="cuda")
    xr = torch.empty_like(x)
    ys = [torch.empty((M, 1024), dtype=torch.float16, device="cuda") for _ in range(2)]
    hr = torch.empty_like(x)
    out = torch.empty((M, 1024), dtype=torch.float16, device="cuda")

    def step():
        api.rotate(x, R1d, out=xr)
        api.linear_group(xr, ws, outs=ys)
        api.rotate(ys[0], R1d, out=hr)
        api.linear(hr, ws[1], out=out)

    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        step()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step()
    for rep in range(2):
        xh = synth.draw_x(rng, M, K)
        x.copy_(torch.from_numpy(xh))
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        a = oracle.round_fp16(oracle.rotate(xh, R1))
        y0 = oracle.round_fp16(oracle.linear(a, ts[0].T1, ts[0].s1, ts[0].res_rows, ts[0].T2, ts[0].s2))
        y1 = oracle.linear(a, ts[1].T1, ts[1].s1, ts[1].res_rows, ts[1].T2, ts[1].s2)
        b = oracle.round_fp16(oracle.rotate(y0, R1))
        y2 = oracle.linear(b, ts[1].T1, ts[1].s1, ts[1].res_rows, ts[1].T2, ts[1].s2)
        assert oracle.rel_err(ys[1].cpu().numpy().astype(np.float64), y1) <= TOL
        assert oracle.rel_err(out.cpu().numpy().astype(np.float64), y2) <= 5e-3
    del g
