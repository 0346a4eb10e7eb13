"""GPU parity of the element-level second plane against the oracle.

* tern_pack_elem / tern_unpack_elem: bit-exact against the oracle's packing, on ragged shapes and
  densities from 0 to 1, with invalid trits and inconsistent metadata reported;
* tern_weight_validate on element planes;
* tern_linear with an element plane: max|y - y_ref| / max|y_ref| <= 2e-3 on seeded inputs at
  M from 1 to 300 (decode GEMV and prefill GEMM), with and without an offset, at densities that
  take both the staged and the global path of the decode kernel; bit-exact where fp32
  accumulation is exact; equal to the row-residual form when the plane covers whole rows; the
  8B gate at full size for M = 1, 16 and 2048 on sampled columns.
"""

import numpy as np
import pytest
import torch

import oracle
from ternary_weight_only_tern_b200 import _lib, api, synth

pytestmark = pytest.mark.gpu
TOL = 2e-3


def _empty_res(K):
    return np.zeros(0, np.int32), np.zeros((0, K), np.int8), np.zeros((0, K // 128), np.float16)


def _trits_at(rng, shape, density):
    return np.where(rng.random(shape) < density, synth.draw_trits(rng, shape, 0.4), 0).astype(np.int8)


@pytest.mark.parametrize("N,K,density", [(1, 128, 0.05), (63, 256, 0.036), (64, 128, 0.0), (65, 384, 0.036),
                                         (130, 128, 1.0), (1000 + 7, 1152, 0.5), (4096, 2560, 0.036)])
def test_pack_elem_matches_oracle(N, K, density):
    rng = np.random.default_rng(N + K)
    T = np.where(rng.random((N, K)) < density, rng.choice(np.array([-1, 1], np.int8), (N, K)), 0).astype(np.int8)
    c, b, e, _ = oracle.pack_elem(T)
    p = api.pack_elem(torch.from_numpy(T).cuda())
    assert p.nnz2 == len(e)
    assert np.array_equal(p.ecount.cpu().numpy(), c)
    assert np.array_equal(p.ebase.cpu().numpy().astype(np.int64), b)
    got = p.eidx.cpu().numpy()
    assert np.array_equal(got[:p.nnz2], e) and not got[p.nnz2:].any()     # padding zeroed
    assert np.array_equal(api.unpack_elem(p).cpu().numpy(), T)


def test_pack_elem_reports_invalid_trits():
    T = np.zeros((3, 128), np.int8)
    T[0, 5], T[1, 9], T[2, 0] = 2, -7, 1
    t = torch.from_numpy(T).cuda()
    with pytest.raises(_lib.TernError) as ei:
        api.pack_elem(t)
    assert ei.value.name == "TERN_ERR_BAD_TRIT"


def test_unpack_and_validate_flag_inconsistent_metadata():
    T, cnt, base, idx = (np.zeros((2, 256), np.int8), np.array([[1, 2], [1, 1]], np.uint8), np.array([0, 3, 5]),
                         np.array([6, 1, 254, 5, 254], np.uint8))
    T[0, 3], T[0, 130], T[1, 0], T[1, 127], T[1, 255] = 1, -1, -1, 1, 1

    def plane(c, b, i):
        e = np.zeros(16, np.uint8)
        e[:len(i)] = i
        return api.ElemPlane(2, 256, torch.from_numpy(c).cuda().contiguous(),
                             torch.from_numpy(b.astype(np.int32)).cuda(), torch.from_numpy(e).cuda(), len(i))

    assert np.array_equal(api.unpack_elem(plane(cnt, base, idx)).cpu().numpy(), T)
    bad_cases = [(cnt, base, idx[[0, 2, 1, 3, 4]]),                      # k not increasing
                 (np.array([[1, 1], [1, 1]], np.uint8), base, idx),     # block sum != base gap
                 (cnt, np.array([1, 3, 5]), idx),                        # ebase[0] != 0
                 (cnt, np.array([0, 3, 4]), idx[:4]),                    # block sum != base gap (last)
                 (np.array([[200, 2], [1, 1]], np.uint8), base, idx)]    # count above 128
    for c, b, i in bad_cases:
        with pytest.raises(_lib.TernError) as ei:
            api.unpack_elem(plane(c, b, i))
        assert ei.value.name == "TERN_ERR_ELEM"
    # the same checks through tern_weight_validate
    rng = np.random.default_rng(1)
    T1 = synth.draw_trits(rng, (2, 256), 0.4)
    s1 = synth.draw_scales(rng, 2, 256, 0.005, 0.02)
    w = api.TernWeight.from_numpy(T1, s1, *_empty_res(256), T2e=T, s2e=synth.draw_scales(rng, 2, 256, 0.001, 0.005))
    api.weight_validate(w)
    wb = api.TernWeight(w.N, w.K, w.plane1, w.scale1, w.res_rows, w.res_slot, w.plane2, w.scale2,
                        elem=plane(cnt, base, idx[[0, 2, 1, 3, 4]]), escale=w.escale)
    with pytest.raises(_lib.TernError) as ei:
        api.weight_validate(wb)
    assert ei.value.name == "TERN_ERR_ELEM"


def _weight(t, T2e, s2e, mu=None):
    return api.TernWeight.from_numpy(t.T1, t.s1, *_empty_res(t.K), mu=mu, T2e=T2e, s2e=s2e)


def _run(w, x):
    y = api.linear(torch.from_numpy(np.ascontiguousarray(x)).cuda(), w)
    torch.cuda.synchronize()
    return y.cpu().numpy()


def _check(y, y_ref):
    assert np.isfinite(y).all()
    err = oracle.rel_err(y.astype(np.float64), y_ref)
    assert err <= TOL, f"rel err {err:.3e}"


@pytest.mark.parametrize("with_mu", [False, True])
@pytest.mark.parametrize("N,K,density", [(320, 1152, 0.036), (1000 + 7, 12288, 0.036), (64, 128, 1.0),
                                         (256, 2560, 0.5)])
def test_elem_linear_parity(N, K, density, with_mu):
    rng = np.random.default_rng(N + K + int(with_mu))
    t = synth.draw_tensor(rng, "elem", N, K, 300, p_zero=0.4, res_pct=0)
    T2e = _trits_at(rng, (N, K), density)
    s2e = synth.draw_scales(rng, N, K, 0.001, 0.005)
    mu = synth.draw_offsets(rng, N, K) if with_mu else None
    w = _weight(t, T2e, s2e, mu)
    y_ref = oracle.linear(t.x, t.T1, t.s1, *_empty_res(K), mu=mu, elem=(T2e, s2e))
    for M in (1, 2, 5, 8, 9, 16, 17, 300):
        _check(_run(w, t.x[:M]), y_ref[:M])


@pytest.mark.parametrize("M", [1, 4, 16, 24, 300])
@pytest.mark.parametrize("N,K,density", [(256, 512, 0.036), (130, 12288, 0.1), (64, 256, 1.0)])
def test_elem_exact_case_bit_exact(M, N, K, density):
    rng = np.random.default_rng(M + N + K)
    t = synth.draw_exact_tensor(rng, N, K, M, 0)
    T2e = _trits_at(rng, (N, K), density)
    s2e = np.ldexp(1.0, -rng.integers(4, 7, size=(N, K // 128))).astype(np.float16)
    y = _run(_weight(t, T2e, s2e), t.x)
    y_ref = oracle.round_fp16(oracle.linear(t.x, t.T1, t.s1, *_empty_res(K), elem=(T2e, s2e)))
    assert np.array_equal(y.view(np.uint16), y_ref.view(np.uint16))


@pytest.mark.parametrize("M", [1, 7, 16, 40])
def test_elem_plane_on_whole_rows_gives_the_row_residual_bits(M):
    """On exact inputs, an element plane covering whole rows R gives the row-residual form's bits."""
    rng = np.random.default_rng(40 + M)
    t = synth.draw_exact_tensor(rng, 300, 1024, M, 31)
    T2e = np.zeros((t.N, t.K), np.int8)
    T2e[t.res_rows] = t.T2
    s2e = np.ldexp(1.0, -rng.integers(4, 7, size=(t.N, t.K // 128))).astype(np.float16)
    s2e[t.res_rows] = t.s2
    w_row = api.TernWeight.from_numpy(t.T1, t.s1, t.res_rows, t.T2, t.s2)
    y_row = _run(w_row, t.x)
    y_elem = _run(_weight(t, T2e, s2e), t.x)
    assert np.array_equal(y_row.view(np.uint16), y_elem.view(np.uint16))


@pytest.mark.parametrize("M", [1, 16, 2048])
def test_elem_8b_gate_full_size(M):
    t = next(synth.draw_workload(synth.WORKLOADS[5], only=["gate"]))
    rng = np.random.default_rng(23)
    T2e, s2e, _ = synth.draw_elem_plane(rng, t.N, t.K)
    cols = rng.choice(t.N, 64, replace=False)
    y_ref = oracle.linear(t.x[:M], t.T1, t.s1, *_empty_res(t.K), cols=cols, elem=(T2e, s2e))
    y = _run(_weight(t, T2e, s2e), t.x[:M])
    _check(y[:, cols], y_ref)


@pytest.mark.parametrize("M", [1, 16])
def test_prefetch_of_an_elem_weight_changes_nothing(M):
    rng = np.random.default_rng(3 + M)
    t = synth.draw_tensor(rng, "p", 512, 2560, M, p_zero=0.4, res_pct=0)
    T2e, s2e, _ = synth.draw_elem_plane(rng, t.N, t.K)
    w = _weight(t, T2e, s2e)
    x = torch.from_numpy(t.x).cuda()
    y0 = api.linear(x, w)
    y1 = api.linear(x, w, prefetch=w)
    torch.cuda.synchronize()
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))
    assert _lib.load().tern_device_status(None) == 0
