"""The failure path of the bounded device-side waits, made to run out on purpose without a GPU
fault: a barrier that nothing completes, waited on for about a millisecond. The status word must
report TERN_ERR_TIMEOUT once (and be clear after the read), and the context must stay usable: a
following tern_linear still matches the oracle."""

import numpy as np
import pytest
import torch

import oracle
from ternary_weight_only_tern_b200 import _lib, api, synth

pytestmark = pytest.mark.gpu
S = _lib.STATUS


def test_a_wait_that_runs_out_is_reported_and_the_context_stays_usable():
    lib = _lib.load()
    st = api._stream()
    assert lib.tern_device_status(st) == 0              # clean before
    assert lib.tern_selftest_timeout(1 << 21, st) == 0   # ~1 ms at the B200's clocks
    assert lib.tern_device_status(st) == S["TERN_ERR_TIMEOUT"]
    assert lib.tern_device_status(st) == 0              # the read cleared it
    rng = np.random.default_rng(9)
    for M in (1, 5, 40):
        t = synth.draw_tensor(rng, "after", 512, 1024, M, p_zero=0.4, res_pct=15)
        w = api.TernWeight.from_numpy(t.T1, t.s1, t.res_rows, t.T2, t.s2)
        y = api.linear(torch.from_numpy(t.x).cuda(), w)
        torch.cuda.synchronize()
        err = oracle.rel_err(y.cpu().numpy().astype(np.float64), oracle.linear(t.x, t.T1, t.s1, t.res_rows, t.T2, t.s2))
        assert err <= 2e-3
    assert lib.tern_device_status(st) == 0


def test_selftest_rejects_bad_bounds():
    lib = _lib.load()
    assert lib.tern_selftest_timeout(0, api._stream()) == S["TERN_ERR_SHAPE"]
    assert lib.tern_selftest_timeout((1 << 32) + 1, api._stream()) == S["TERN_ERR_SHAPE"]
