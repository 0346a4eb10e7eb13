"""GPU parity of tern_fit (dense W to ternary planes, scales and offset) against the oracle.

The fit's decisions (thresholds, planes) and its scales are compared bit for bit: both sides run the
same float64 operations in the same order and round each scale once. Covered: ragged shapes, with
and without an offset and residual rows, 0, 1 and 15 refinement rounds, zero and constant groups,
a hand-worked group, the 8B gate at full size (sampled rows), and the fitted planes through
tern_linear against the oracle's product.
"""

import numpy as np
import pytest
import torch

import oracle
from ternary_weight_only_tern_b200 import api, synth

pytestmark = pytest.mark.gpu


def _fit(W, rows, offset=True, iters=15):
    out = api.fit(torch.from_numpy(W).cuda(), torch.from_numpy(rows).cuda(), offset=offset, iters=iters)
    torch.cuda.synchronize()
    return [None if t is None else t.cpu().numpy() for t in out]


def _same(got, ref):
    T1, s1, mu, T2, s2 = got
    R1, r1, rm, R2, r2 = ref
    assert np.array_equal(T1, R1) and np.array_equal(T2, R2)
    assert np.array_equal(s1.view(np.uint16), r1.view(np.uint16))
    assert np.array_equal(s2.view(np.uint16), r2.view(np.uint16))
    assert (mu is None) == (rm is None)
    if mu is not None:
        assert np.array_equal(mu.view(np.uint16), rm.view(np.uint16))


@pytest.mark.parametrize("offset", [True, False])
@pytest.mark.parametrize("iters", [0, 1, 15])
@pytest.mark.parametrize("N,K,pct", [(70, 384, 10), (1000 + 7, 1152, 15), (3, 128, 100)])
def test_fit_matches_oracle_bit_for_bit(N, K, pct, offset, iters):
    rng = np.random.default_rng(N + K + iters + int(offset))
    W = (rng.standard_normal((N, K)) * 0.02 + rng.uniform(-0.005, 0.005, (N, 1))).astype(np.float16)
    W[0, :128] = 0                     # a zero group
    W[-1, -128:] = np.float16(0.0625)  # a constant group
    rows = np.sort(rng.choice(N, synth.residual_count(N, pct), replace=False)).astype(np.int32)
    _same(_fit(W, rows, offset, iters), oracle.ternarize(W, rows, offset=offset, iters=iters))


def test_fit_hand_worked_group():
    w = np.array([1.0] * 64 + [0.4] * 64, dtype=np.float16)[None]
    T1, s1, mu, T2, s2 = _fit(w, np.array([0], np.int32), offset=False)
    assert np.array_equal(T1[0], [1] * 64 + [0] * 64) and np.array_equal(T2[0], [0] * 64 + [1] * 64)
    assert s1[0, 0] == 1.0 and s2[0, 0] == np.float16(0.4) and mu is None


def test_fit_8b_gate_full_size_sampled_rows():
    rng = np.random.default_rng(77)
    N, K = synth.QWEN3_8B["gate"]
    W = (rng.standard_normal((N, K), dtype=np.float32) * 0.02).astype(np.float16)
    rows = np.sort(rng.choice(N, synth.residual_count(N, 15), replace=False)).astype(np.int32)
    T1, s1, mu, T2, s2 = _fit(W, rows)
    pick = np.sort(np.concatenate([rng.choice(N, 96, replace=False), rows[:32]]))
    pick = np.unique(pick)
    sub_rows = np.array([i for i, n in enumerate(pick) if n in set(rows.tolist())], np.int32)
    R1, r1, rm, R2, r2 = oracle.ternarize(W[pick], sub_rows)
    slot = {int(n): i for i, n in enumerate(rows)}
    assert np.array_equal(T1[pick], R1) and np.array_equal(s1[pick].view(np.uint16), r1.view(np.uint16))
    assert np.array_equal(mu[pick].view(np.uint16), rm.view(np.uint16))
    gpu_slots = [slot[int(pick[i])] for i in sub_rows]
    assert np.array_equal(T2[gpu_slots], R2) and np.array_equal(s2[gpu_slots].view(np.uint16), r2.view(np.uint16))


@pytest.mark.parametrize("M", [1, 16, 40])
def test_fitted_weight_through_tern_linear(M):
    """fit -> pack -> tern_linear equals the oracle's product with the oracle's fit of the same W."""
    rng = np.random.default_rng(5 + M)
    N, K = 1000 + 7, 2560
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    rows = np.sort(rng.choice(N, synth.residual_count(N, 10), replace=False)).astype(np.int32)
    Wd = torch.from_numpy(W).cuda()
    T1, s1, mu, T2, s2 = api.fit(Wd, torch.from_numpy(rows).cuda())
    w = api.TernWeight.from_trits(T1, s1, torch.from_numpy(rows).cuda(), T2, s2, mu=mu)
    x = synth.draw_x(rng, M, K)
    y = api.linear(torch.from_numpy(x).cuda(), w)
    torch.cuda.synchronize()
    R1, r1, rm, R2, r2 = oracle.ternarize(W, rows)
    y_ref = oracle.linear(x, R1, r1, rows, R2, r2, mu=rm)
    assert oracle.rel_err(y.cpu().numpy().astype(np.float64), y_ref) <= 2e-3
