"""The C-ABI library loads and exports every function include/tern.h declares; host-side
logic (bit accounting, argument validation) needs no GPU and is checked here."""

import ctypes
import os
import re

import pytest

import oracle
from ternary_weight_only_tern_b200 import _lib, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    text = open(os.path.join(ROOT, "include", "tern.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tern_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(_lib.LIB_PATH):
        from ternary_weight_only_tern_b200 import build
        build.build()
    return _lib.load()


def test_header_declares_the_boundary():
    fns = header_functions()
    for name in ["tern_pack_exec", "tern_unpack_exec", "tern_pack_store", "tern_unpack_store",
                 "tern_linear_workspace_bytes", "tern_linear", "tern_linear_with_prefetch", "tern_bits",
                 "tern_status_string"]:
        assert name in fns
    assert set(fns) == set(_lib.EXPORTS), "ctypes declarations and header disagree"


def test_library_exports_every_declared_symbol(lib):
    for name in header_functions():
        assert hasattr(lib, name), name
    assert lib.tern_version() >= 100


def test_status_strings(lib):
    for code in range(12):
        assert lib.tern_status_string(code)
    assert lib.tern_status_string(99) == b"unknown status"


def test_release_and_debug_builds_identify_themselves(lib):
    """The TERN_DEBUG build (libtern_debug.so) exports the same boundary and says it is the debug
    build; the release build says it is not; TERN_LIBRARY=debug loads the debug build."""
    assert lib.tern_debug_build() == (1 if os.environ.get("TERN_LIBRARY") == "debug" else 0)
    path = os.path.join(os.path.dirname(_lib.LIB_PATH), "libtern_debug.so")
    if not os.path.exists(path):
        from ternary_weight_only_tern_b200 import build
        build.build(debug=True)
    dbg = ctypes.CDLL(path)
    for name in header_functions():
        assert hasattr(dbg, name), name
    dbg.tern_debug_build.restype = ctypes.c_int
    assert dbg.tern_debug_build() == 1


@pytest.mark.parametrize("N,K,r", [(4096, 2560, 0), (9728, 2560, 973), (12288, 4096, 1843), (13, 384, 13),
                                   (1024, 12288, 154), (1, 128, 1)])
def test_tern_bits_equals_oracle(lib, N, K, r):
    rep = _lib.TernBitsReport()
    assert lib.tern_bits(N, K, r, 128, ctypes.byref(rep)) == 0
    ref = oracle.bits(N, K, r)
    for f in ("weights", "plane_trits", "store_bits", "exec_bits"):
        assert getattr(rep, f) == ref[f], f
    for f in ("bpw_info", "bpw_store", "bpw_exec"):
        assert getattr(rep, f) == pytest.approx(ref[f], rel=1e-15, abs=0), f


@pytest.mark.parametrize("N,K,r", [(4096, 2560, 0), (12288, 4096, 1843), (1, 128, 1)])
def test_tern_bits_offset_equals_oracle(lib, N, K, r):
    rep = _lib.TernBitsReport()
    assert lib.tern_bits_offset(N, K, r, 128, ctypes.byref(rep)) == 0
    ref = oracle.bits(N, K, r, offset=True)
    for f in ("weights", "plane_trits", "store_bits", "exec_bits"):
        assert getattr(rep, f) == ref[f], f
    for f in ("bpw_info", "bpw_store", "bpw_exec"):
        assert getattr(rep, f) == pytest.approx(ref[f], rel=1e-15, abs=0), f
    assert lib.tern_bits_offset(16, 100, 0, 128, ctypes.byref(rep)) == _lib.STATUS["TERN_ERR_SHAPE"]


def test_tern_bits_whole_stack(lib):
    # the 252 targeted tensors of the 4B model at 10% residual rows: sum of per-tensor integers
    rep = _lib.TernBitsReport()
    tot = {"weights": 0, "store_bits": 0, "exec_bits": 0}
    for (_, N, K) in synth.WORKLOADS[3].shapes:
        r = synth.residual_count(N, 10)
        assert lib.tern_bits(N, K, r, 128, ctypes.byref(rep)) == 0
        for k in tot:
            tot[k] += synth.N_LAYERS * getattr(rep, k)
    assert tot["weights"] == 3_633_315_840       # = 36 * (4096+2048)*2560 + 2560*4096 + 3*9728*2560 ...
    assert 1.7 < tot["store_bits"] / tot["weights"] < 2.0


def test_tern_bits_rejects(lib):
    rep = _lib.TernBitsReport()
    S = _lib.STATUS
    assert lib.tern_bits(0, 128, 0, 128, ctypes.byref(rep)) == S["TERN_ERR_SHAPE"]
    assert lib.tern_bits(16, 100, 0, 128, ctypes.byref(rep)) == S["TERN_ERR_SHAPE"]
    assert lib.tern_bits(16, 128, 0, 64, ctypes.byref(rep)) == S["TERN_ERR_SHAPE"]
    assert lib.tern_bits(16, 128, 17, 128, ctypes.byref(rep)) == S["TERN_ERR_SHAPE"]
    assert lib.tern_bits(16, 128, 0, 128, None) == S["TERN_ERR_NULL"]


def test_linear_host_validation(lib):
    """Every check here fails before a launch, so no device is touched."""
    S = _lib.STATUS
    fake = 1 << 20         # an aligned non-null address that is never dereferenced on these paths
    w = _lib.TernWeightC(64, 256, 128, fake, fake, 0, None, fake, None, None, 0)
    call = lambda w, x, M, y, ws=None, wsb=0: lib.tern_linear(  # noqa: E731
        ctypes.byref(w) if w is not None else None, x, M, y, ws, wsb, None)
    assert call(None, fake, 1, fake) == S["TERN_ERR_NULL"]
    assert call(w, fake, 0, fake) == S["TERN_OK"]                 # M == 0 is a no-op
    assert call(w, None, 1, fake) == S["TERN_ERR_NULL"]
    assert call(w, fake + 2, 1, fake * 4) == S["TERN_ERR_ALIGN"]
    assert call(w, fake, 1, fake) == S["TERN_ERR_SHAPE"]          # x and y overlap
    assert call(w, fake, -1, fake) == S["TERN_ERR_SHAPE"]
    bad = _lib.TernWeightC(64, 200, 128, fake, fake, 0, None, fake, None, None, 0)
    assert call(bad, fake, 1, fake * 4) == S["TERN_ERR_SHAPE"]
    bad = _lib.TernWeightC(64, 256, 64, fake, fake, 0, None, fake, None, None, 0)
    assert call(bad, fake, 1, fake * 4) == S["TERN_ERR_SHAPE"]
    bad = _lib.TernWeightC(64, 256, 128, fake, fake, 65, fake, fake, fake, fake, 0)
    assert call(bad, fake, 1, fake * 4) == S["TERN_ERR_SHAPE"]    # r > N
    bad = _lib.TernWeightC(64, 256, 128, fake, fake, 4, fake, fake, None, fake, 0)
    assert call(bad, fake, 1, fake * 4) == S["TERN_ERR_NULL"]     # residual plane missing
    bad = _lib.TernWeightC(64, 256, 128, fake + 4, fake, 0, None, fake, None, None, 0)
    assert call(bad, fake, 1, fake * 4) == S["TERN_ERR_ALIGN"]
    bad = _lib.TernWeightC(64, 256, 128, fake, fake, 0, None, fake, None, None, 0, fake + 2)
    assert call(bad, fake, 1, fake * 4) == S["TERN_ERR_ALIGN"]    # misaligned offset
    # element plane: exclusive with residual rows, its arrays non-null and aligned
    E = lambda r=0, ec=fake, eb=fake, ei=fake, es=fake, nnz=5: _lib.TernWeightC(  # noqa: E731
        64, 256, 128, fake, fake, r, fake if r else None, fake, fake if r else None, fake if r else None, 0, None,
        ec, eb, ei, es, nnz)
    assert call(E(r=4), fake, 1, fake * 4) == S["TERN_ERR_SHAPE"]
    assert call(E(nnz=-1), fake, 1, fake * 4) == S["TERN_ERR_SHAPE"]
    assert call(E(eb=None), fake, 1, fake * 4) == S["TERN_ERR_NULL"]
    assert call(E(es=None), fake, 1, fake * 4) == S["TERN_ERR_NULL"]
    assert call(E(ei=None), fake, 1, fake * 4) == S["TERN_ERR_NULL"]
    assert call(E(ec=fake + 1), fake, 1, fake * 4) == S["TERN_ERR_ALIGN"]
    assert call(E(ei=fake + 8), fake, 1, fake * 4) == S["TERN_ERR_ALIGN"]
    assert call(E(), fake, 0, fake) == S["TERN_OK"]
    # neither path needs scratch memory
    wr = _lib.TernWeightC(64, 256, 128, fake, fake, 4, fake, fake, fake, fake, 1)
    for M in (1, 16, 17, 4096):
        assert lib.tern_linear_workspace_bytes(ctypes.byref(wr), M) == 0
    assert call(wr, fake + 2, 3, fake * 4) == S["TERN_ERR_ALIGN"]
    assert call(wr, fake, 3, fake * 4, fake * 8 + 4, 64) == S["TERN_ERR_ALIGN"]   # misaligned workspace
    # the prefetch descriptor is checked like the weight; a good one changes nothing up to the launch
    pf = lambda nxt, M=1: lib.tern_linear_with_prefetch(  # noqa: E731
        ctypes.byref(w), fake, M, fake * 4, None, 0, ctypes.byref(nxt) if nxt is not None else None, None)
    assert pf(_lib.TernWeightC(64, 200, 128, fake, fake, 0, None, fake, None, None, 0)) == S["TERN_ERR_SHAPE"]
    assert pf(_lib.TernWeightC(64, 256, 128, fake + 4, fake, 0, None, fake, None, None, 0)) == S["TERN_ERR_ALIGN"]
    assert pf(_lib.TernWeightC(64, 256, 128, fake, fake, 4, fake, fake, None, fake, 0)) == S["TERN_ERR_NULL"]
    assert pf(w, M=0) == S["TERN_OK"]
    assert pf(None, M=0) == S["TERN_OK"]


@pytest.mark.parametrize("N,K,masked,nnz2,offset", [(4096, 2560, 377487, 226492, 0), (13, 384, 250, 140, 1),
                                                     (12288, 4096, 0, 0, 0)])
def test_tern_bits_elem_equals_oracle(lib, N, K, masked, nnz2, offset):
    rep = _lib.TernBitsReport()
    assert lib.tern_bits_elem(N, K, masked, nnz2, 128, offset, ctypes.byref(rep)) == 0
    ref = oracle.bits_elem(N, K, masked, nnz2, offset=bool(offset))
    for f in ("weights", "plane_trits", "store_bits", "exec_bits"):
        assert getattr(rep, f) == ref[f], f
    for f in ("bpw_info", "bpw_store", "bpw_exec"):
        assert getattr(rep, f) == pytest.approx(ref[f], rel=1e-15, abs=0), f
    S = _lib.STATUS
    assert lib.tern_bits_elem(N, K, masked, masked + 1, 128, 0, ctypes.byref(rep)) == S["TERN_ERR_SHAPE"]
    assert lib.tern_bits_elem(N, K, N * K + 1, 0, 128, 0, ctypes.byref(rep)) == S["TERN_ERR_SHAPE"]
    assert lib.tern_bits_elem(N, K, masked, nnz2, 128, 0, None) == S["TERN_ERR_NULL"]


def test_elem_pack_host_validation(lib):
    """Checks that fail before any launch."""
    S = _lib.STATUS
    fake = 1 << 20
    nnz = ctypes.c_int64(7)
    assert lib.tern_pack_elem(fake, 4, 128, fake, fake, None, 0, None, None) == S["TERN_ERR_NULL"]
    assert lib.tern_pack_elem(fake, 4, 100, fake, fake, None, 0, ctypes.byref(nnz), None) == S["TERN_ERR_SHAPE"]
    assert nnz.value == 0
    assert lib.tern_pack_elem(fake, -1, 128, fake, fake, None, 0, ctypes.byref(nnz), None) == S["TERN_ERR_SHAPE"]
    assert lib.tern_pack_elem(fake, 4, 128, fake, None, None, 0, ctypes.byref(nnz), None) == S["TERN_ERR_NULL"]
    assert lib.tern_pack_elem(fake, 4, 128, fake, fake + 4, None, 0, ctypes.byref(nnz), None) == S["TERN_ERR_ALIGN"]
    assert lib.tern_pack_elem(None, 4, 128, fake, fake, None, 0, ctypes.byref(nnz), None) == S["TERN_ERR_NULL"]
    assert lib.tern_pack_elem(fake + 1, 4, 128, fake, fake, None, 0, ctypes.byref(nnz), None) == S["TERN_ERR_ALIGN"]
    assert lib.tern_unpack_elem(fake, fake, fake, 3, 4, 100, fake, None) == S["TERN_ERR_SHAPE"]
    assert lib.tern_unpack_elem(fake, fake, fake, -1, 4, 128, fake, None) == S["TERN_ERR_SHAPE"]
    assert lib.tern_unpack_elem(fake, fake, None, 3, 4, 128, fake, None) == S["TERN_ERR_NULL"]
    assert lib.tern_unpack_elem(fake, fake + 4, fake, 3, 4, 128, fake, None) == S["TERN_ERR_ALIGN"]
    assert lib.tern_unpack_elem(fake, fake, fake, 3, 0, 128, fake, None) == S["TERN_OK"]


def test_linear_group_host_validation(lib):
    """Checks of tern_linear_group that fail before a launch."""
    S = _lib.STATUS
    fake = 1 << 20
    mk = lambda N=64, K=256, ec=None: _lib.TernWeightC(64 if N is None else N, K, 128, fake, fake, 0, None, fake,  # noqa
                                                        None, None, 0, None, ec, fake if ec else None,
                                                        fake if ec else None, fake if ec else None, 0)
    w1, w2 = mk(), mk(N=32)
    arr = lambda *ws: (ctypes.c_void_p * len(ws))(*[ctypes.addressof(w) for w in ws])  # noqa: E731
    ys = lambda *ps: (ctypes.c_void_p * len(ps))(*ps)  # noqa: E731
    g = lambda w, n, M, y, x=fake: lib.tern_linear_group(w, n, x, M, y, None, 0, None, 0, None)  # noqa: E731
    Y = ys(fake * 4, fake * 8)
    assert g(arr(w1, w2), 0, 1, Y) == S["TERN_ERR_SHAPE"]
    assert g(arr(w1, w2, w1, w2, w1), 5, 1, ys(*[fake * 4] * 5)) == S["TERN_ERR_SHAPE"]
    assert g(None, 2, 1, Y) == S["TERN_ERR_NULL"]
    assert g(arr(w1, w2), 2, 1, None) == S["TERN_ERR_NULL"]
    assert g(arr(w1, mk(K=384)), 2, 1, Y) == S["TERN_ERR_SHAPE"]                  # K differs
    assert g(arr(w1, mk(ec=fake)), 2, 1, Y) == S["TERN_ERR_SHAPE"]                # element plane on one only
    assert g(arr(w1, w2), 2, 1, ys(fake * 4, fake * 4 + 64)) == S["TERN_ERR_SHAPE"]   # outputs overlap
    assert g(arr(w1, w2), 2, 1, ys(fake * 4, fake)) == S["TERN_ERR_SHAPE"]        # an output overlaps x
    assert g(arr(w1, w2), 2, 1, ys(fake * 4, fake * 8 + 2)) == S["TERN_ERR_ALIGN"]
    assert g(arr(w1, w2), 2, 1, ys(fake * 4, None)) == S["TERN_ERR_NULL"]
    assert g(arr(w1, w2), 2, 0, Y) == S["TERN_OK"]                                # M == 0 is a no-op
    assert lib.tern_linear_group(arr(w1, w2), 2, fake, 1, Y, None, 0, None, 1, None) == S["TERN_ERR_NULL"]
    assert lib.tern_linear_group(arr(w1, w2), 2, fake, 1, Y, None, 0, arr(mk(K=100)), 1, None) == S["TERN_ERR_SHAPE"]


def test_fit_host_validation(lib):
    S = _lib.STATUS
    f = 1 << 20
    fit = lambda W=f, N=4, K=256, slot=None, r=0, off=1, it=15, T1=f * 2, s1=f * 3, mu=f * 4, T2=None, s2=None: \
        lib.tern_fit(W, N, K, slot, r, off, it, T1, s1, mu, T2, s2, None)  # noqa: E731
    assert fit(K=200) == S["TERN_ERR_SHAPE"]
    assert fit(r=5) == S["TERN_ERR_SHAPE"]
    assert fit(it=-1) == S["TERN_ERR_SHAPE"]
    assert fit(N=0) == S["TERN_OK"]
    assert fit(W=None) == S["TERN_ERR_NULL"]
    assert fit(mu=None) == S["TERN_ERR_NULL"]                   # an offset needs mu
    assert fit(r=2, slot=f * 5) == S["TERN_ERR_NULL"]           # residual rows need T2 and s2
    assert fit(W=f + 2) == S["TERN_ERR_ALIGN"]
    assert fit(T1=f * 2 + 8) == S["TERN_ERR_ALIGN"]


def test_rotate_host_validation(lib):
    S = _lib.STATUS
    fake = 1 << 20
    assert lib.tern_rotate(fake, 4, 100, fake * 2, fake * 4, None) == S["TERN_ERR_SHAPE"]
    assert lib.tern_rotate(fake, -1, 128, fake * 2, fake * 4, None) == S["TERN_ERR_SHAPE"]
    assert lib.tern_rotate(fake, 0, 128, None, None, None) == S["TERN_OK"]
    assert lib.tern_rotate(None, 4, 128, fake * 2, fake * 4, None) == S["TERN_ERR_NULL"]
    assert lib.tern_rotate(fake, 4, 128, None, fake * 4, None) == S["TERN_ERR_NULL"]
    assert lib.tern_rotate(fake + 2, 4, 128, fake * 2, fake * 4, None) == S["TERN_ERR_ALIGN"]
    assert lib.tern_rotate(fake, 4, 128, fake * 2 + 8, fake * 4, None) == S["TERN_ERR_ALIGN"]
    assert lib.tern_rotate(fake, 4, 128, fake * 2, fake + 256, None) == S["TERN_ERR_SHAPE"]   # x, y overlap


def test_pack_host_validation(lib):
    S = _lib.STATUS
    fake = 1 << 20
    assert lib.tern_pack_exec(fake, 4, 17, fake * 2, None) == S["TERN_ERR_SHAPE"]
    assert lib.tern_pack_exec(None, 4, 16, fake, None) == S["TERN_ERR_NULL"]
    assert lib.tern_pack_exec(fake + 1, 4, 16, fake * 2, None) == S["TERN_ERR_ALIGN"]
    assert lib.tern_pack_exec(fake, 0, 16, fake * 2, None) == S["TERN_OK"]
    assert lib.tern_unpack_exec(fake, -1, 16, fake * 2, None) == S["TERN_ERR_SHAPE"]
    assert lib.tern_pack_store(None, 4, 7, fake, None) == S["TERN_ERR_NULL"]
    assert lib.tern_unpack_store(fake, 4, -7, fake, None) == S["TERN_ERR_SHAPE"]
    assert lib.tern_weight_validate(None, None) == S["TERN_ERR_NULL"]


def test_binding_caches_follow_the_weight(lib):
    """The binding remembers a weight's C descriptor, its workspace sizes and a group's pointer
    array; changing a field of the weight must give a fresh descriptor (host logic only: the
    tensors stay on the host and no kernel runs)."""
    import torch
    from ternary_weight_only_tern_b200 import api

    N, K = 64, 256

    def weight():
        return api.TernWeight(N, K, torch.zeros((N, K // 16), dtype=torch.int32),
                              torch.zeros((N, K // 128), dtype=torch.float16),
                              torch.zeros(0, dtype=torch.int32), torch.full((N,), -1, dtype=torch.int32),
                              torch.zeros((0, K // 16), dtype=torch.int32),
                              torch.zeros((0, K // 128), dtype=torch.float16))

    w, v = weight(), weight()
    c1 = w.c_struct()
    assert c1 is w.c_struct() and c1.flags == 0
    w.static = True
    c2 = w.c_struct()
    assert c2 is not c1 and c2.flags == _lib.WEIGHT_STATIC and c2.N == N and c2.K == K
    assert api.workspace_bytes(w, 1) == lib.tern_linear_workspace_bytes(ctypes.byref(c2), 1)
    assert 1 in w._ws
    a1 = api._weight_array([w, v])
    assert a1 is api._weight_array([w, v])
    assert [a1[0], a1[1]] == [ctypes.addressof(w.c_struct()), ctypes.addressof(v.c_struct())]
    v.static = True                       # a new descriptor for v: a new array
    a2 = api._weight_array([w, v])
    assert a2 is not a1 and a2[1] == ctypes.addressof(v.c_struct())
    assert w._ws is not None and v._ws is None


def _ranges_cost(ranges, strips, Sb, nstage, seg_strips=16):
    """Per-CTA stages of a split, on the kernels' walk: each CTA's strips in segments (one weight,
    at most seg_strips strips, from the CTA's first strip), each ceil(main / Sb) blocks of main
    strips and ceil(ceil(residual rows / 16) / Sb) of residual strips, nstage stages a block.
    strips: [(weight, residual rows)] of the launch in order. Also the segment counts."""
    costs, segs = [], []
    for a, b in zip(ranges[:-1], ranges[1:]):
        c, ns, j = 0, 0, a
        while j < b:
            e = j
            while e < b and strips[e][0] == strips[j][0] and e - j < seg_strips:
                e += 1
            rows = sum(strips[k][1] for k in range(j, e))
            c += (-(-(e - j) // Sb) + -(-(-(-rows // 16)) // Sb)) * nstage
            ns += 1
            j = e
        costs.append(c)
        segs.append(ns)
    return costs, segs


def test_decode_ranges_balance_residual_strips(lib):
    """tern_decode_ranges on host descriptors: without res_per_strip the even split
    [b S / P, (b + 1) S / P); with it a split that covers every strip in order, keeps each CTA
    within 8 segments, and whose slowest CTA walks no more stages than the even split's, strictly
    fewer when the residual rows are bunched at one end (gate and up of the 8B model)."""
    import dataclasses
    import numpy as np
    import torch
    from ternary_weight_only_tern_b200 import api

    N, K, r = 12288, 4096, 1843
    rng = np.random.default_rng(11)
    ws, strips = [], []
    for i in range(2):
        rows = np.sort(rng.choice(N // 3, size=r, replace=False)).astype(np.int32)   # the first third
        slot = np.full(N, -1, np.int32)
        slot[rows] = np.arange(r, dtype=np.int32)
        hint = torch.from_numpy(np.bincount(rows // 16, minlength=N // 16).astype(np.int16))
        ws.append(api.TernWeight(N, K, torch.zeros((N, K // 16), dtype=torch.int32),
                                 torch.zeros((N, K // 128), dtype=torch.float16), torch.from_numpy(rows),
                                 torch.from_numpy(slot), torch.zeros((r, K // 16), dtype=torch.int32),
                                 torch.zeros((r, K // 128), dtype=torch.float16), res_hint=hint))
        strips += [(i, int(c)) for c in hint.numpy()]
    S = len(strips)
    even, Sb, nst = api.decode_ranges([dataclasses.replace(w, res_hint=None) for w in ws], 1)
    P = len(even) - 1
    assert P >= 1 and Sb >= 1 and nst >= 1
    assert even == [b * S // P for b in range(P + 1)]
    bal, Sb2, nst2 = api.decode_ranges(ws, 1)
    assert (Sb2, nst2) == (Sb, nst) and len(bal) == P + 1
    assert bal[0] == 0 and bal[-1] == S and all(x <= y for x, y in zip(bal, bal[1:]))
    ce, _ = _ranges_cost(even, strips, Sb, nst)
    cb, segs = _ranges_cost(bal, strips, Sb, nst)
    assert max(segs) <= 8
    assert max(cb) < max(ce), (max(cb), max(ce))
    # 16 tokens: the multi-token kernel's split, with its own plan
    bal16, Sb16, nst16 = api.decode_ranges(ws, 16)
    even16, _, _ = api.decode_ranges([dataclasses.replace(w, res_hint=None) for w in ws], 16)
    assert bal16[0] == 0 and bal16[-1] == S and len(bal16) == len(even16)
    assert max(_ranges_cost(bal16, strips, Sb16, nst16)[0]) <= max(_ranges_cost(even16, strips, Sb16, nst16)[0])
    # no persistent decode launch past 16 tokens
    assert api.decode_ranges(ws, 17) == ([], 0, 0)


def test_residual_strip_counts(lib):
    """tern_residual_strip_counts equals a per-strip count of the residual rows (ragged N), and
    rejects rows out of range or out of order."""
    import numpy as np

    rng = np.random.default_rng(5)
    for N, r in ((1, 1), (17, 5), (1000 + 9, 150), (12288, 1843)):
        rows = np.sort(rng.choice(N, size=r, replace=False)).astype(np.int32)
        out = np.full((N + 15) // 16, 999, np.uint16)
        st = lib.tern_residual_strip_counts(rows.ctypes.data_as(ctypes.c_void_p), r, N,
                                            out.ctypes.data_as(ctypes.c_void_p))
        assert st == 0
        assert np.array_equal(out, np.bincount(rows // 16, minlength=(N + 15) // 16))
    out = np.zeros(2, np.uint16)
    for bad in (np.array([3, 3], np.int32), np.array([5, 2], np.int32), np.array([0, 20], np.int32)):
        assert lib.tern_residual_strip_counts(bad.ctypes.data_as(ctypes.c_void_p), 2, 20,
                                              out.ctypes.data_as(ctypes.c_void_p)) == 6   # TERN_ERR_RESIDUAL


def test_decode_dispatch_rules(lib):
    """Which decode kernel a call takes, seen through tern_decode_ranges (host descriptors): one
    token and 9-16 tokens always run a persistent kernel; 4-8 tokens only on launches of at least
    10 strips per CTA (the 8B gate and up as one launch), else, like 2-3 tokens, the cluster kernel
    (no split); no persistent kernel past 16 tokens or with an element plane's weights."""
    import torch
    from ternary_weight_only_tern_b200 import api

    def weight(N, K):
        return api.TernWeight(N, K, torch.zeros((N, K // 16), dtype=torch.int32),
                              torch.zeros((N, K // 128), dtype=torch.float16), torch.zeros(0, dtype=torch.int32),
                              torch.full((N,), -1, dtype=torch.int32), torch.zeros((0, K // 16), dtype=torch.int32),
                              torch.zeros((0, K // 128), dtype=torch.float16))

    big = [weight(12288, 4096), weight(12288, 4096)]      # 1536 strips: 11 per CTA
    small = [weight(4096, 4096)]                          # 256 strips: 2 per CTA
    persistent = lambda ws, M: len(api.decode_ranges(ws, M)[0]) > 0  # noqa: E731
    for M in (1, 9, 12, 16):
        assert persistent(big, M) and persistent(small, M), M
    for M in (4, 5, 8):
        assert persistent(big, M) and not persistent(small, M), M
    for M in (2, 3):
        assert not persistent(big, M) and not persistent(small, M), M
    assert not persistent(big, 17)
    import dataclasses
    N, K = 12288, 4096
    G = K // 128
    elem = api.ElemPlane(N, K, torch.zeros((G, N), dtype=torch.uint8), torch.zeros(G * (N // 64) + 1, dtype=torch.int32),
                         torch.zeros(16, dtype=torch.uint8), 0)
    ew = [dataclasses.replace(w, elem=elem, escale=torch.zeros((N, G), dtype=torch.float16)) for w in big]
    for M in (1, 8, 16):
        assert not persistent(ew, M), M


@pytest.mark.parametrize("seed", range(6))
def test_balanced_split_random_groups(lib, seed):
    """Random groups of 1-4 weights (ragged N, 0-100 % residual rows, bunched or spread): the
    balanced split covers every strip in order, keeps each CTA within 8 segments, and its slowest
    CTA walks no more stages than the even split's, for one token and for 16."""
    import dataclasses
    import numpy as np
    import torch
    from ternary_weight_only_tern_b200 import api

    rng = np.random.default_rng(100 + seed)
    K = int(rng.choice([1024, 2048, 4096]))
    ws, strips = [], []
    for i in range(int(rng.integers(1, 5))):
        N = int(rng.integers(1, 9000))
        r = int(rng.integers(0, N + 1)) if rng.random() < 0.8 else 0
        span = N if rng.random() < 0.5 else max(r, N // 4)
        rows = np.sort(rng.choice(span, size=r, replace=False)).astype(np.int32)
        slot = np.full(N, -1, np.int32)
        slot[rows] = np.arange(r, dtype=np.int32)
        hint = None
        if r:
            h = np.zeros((N + 15) // 16, np.uint16)
            assert lib.tern_residual_strip_counts(rows.ctypes.data_as(ctypes.c_void_p), r, N,
                                                  h.ctypes.data_as(ctypes.c_void_p)) == 0
            hint = torch.from_numpy(h.astype(np.int16))
        ws.append(api.TernWeight(N, K, torch.zeros((N, K // 16), dtype=torch.int32),
                                 torch.zeros((N, K // 128), dtype=torch.float16), torch.from_numpy(rows),
                                 torch.from_numpy(slot), torch.zeros((r, K // 16), dtype=torch.int32),
                                 torch.zeros((r, K // 128), dtype=torch.float16), res_hint=hint))
        counts = np.bincount(rows // 16, minlength=(N + 15) // 16) if r else np.zeros((N + 15) // 16, int)
        strips += [(i, int(c)) for c in counts]
    S = len(strips)
    for M in (1, 16):
        bal, Sb, nst = api.decode_ranges(ws, M)
        even, _, _ = api.decode_ranges([dataclasses.replace(w, res_hint=None) for w in ws], M)
        if not bal:
            assert not even
            continue
        assert bal[0] == 0 and bal[-1] == S and len(bal) == len(even)
        assert all(a <= b for a, b in zip(bal, bal[1:]))
        cb, segs = _ranges_cost(bal, strips, Sb, nst)
        ce, _ = _ranges_cost(even, strips, Sb, nst)
        assert max(segs) <= 8
        assert max(cb) <= max(ce), (M, max(cb), max(ce))
