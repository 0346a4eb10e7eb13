"""GPU parity of packing, unpacking and descriptor validation: bit-exact against the oracle."""

import numpy as np
import pytest
import torch

import oracle
from ternary_weight_only_tern_b200 import _lib, api, synth

pytestmark = pytest.mark.gpu
S = _lib.STATUS


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t if dtype is None else t.to(dtype)


def expect_status(fn, *args, status):
    with pytest.raises(_lib.TernError) as e:
        fn(*args)
    assert e.value.status == S[status]


def test_store_all_243_bytes_and_invalid_bytes():
    b = np.arange(256, dtype=np.uint8).reshape(256, 1)
    ref, bad = oracle.unpack_store(b, 5)
    assert bad > 0
    # the valid ones alone decode with TERN_OK
    got = api.unpack_store(dev(b[:243]), 5).cpu().numpy()
    assert np.array_equal(got, ref[:243])
    # with the invalid ones: TERN_ERR_BAD_CODE, and the output still equals the oracle's
    out = torch.empty((256, 5), dtype=torch.int8, device="cuda")
    st = _lib.load().tern_unpack_store(api._ptr(dev(b)), 256, 5, api._ptr(out), api._stream())
    assert st == S["TERN_ERR_BAD_CODE"]
    assert np.array_equal(out.cpu().numpy(), ref)
    # and all 243 valid five-trit tuples pack to their bytes
    combos = ref[:243].copy()
    assert np.array_equal(api.pack_store(dev(combos)).cpu().numpy(), oracle.pack_store(combos)[0])


def test_exec_every_byte_pattern():
    vals = np.arange(256, dtype=np.uint32)
    for pos in range(4):
        words = ((vals << np.uint32(8 * pos)) | np.uint32(0x55555555 & ~(0xFF << (8 * pos)))).reshape(256, 1)
        ref, bad = oracle.unpack_exec(words, 16)
        out = torch.empty((256, 16), dtype=torch.int8, device="cuda")
        st = _lib.load().tern_unpack_exec(api._ptr(dev(words.view(np.int32))), 256, 16, api._ptr(out), api._stream())
        assert st == S["TERN_ERR_BAD_CODE"] and bad > 0
        assert np.array_equal(out.cpu().numpy(), ref)


@pytest.mark.parametrize("shape", sorted({(N, K) for w in synth.WORKLOADS.values() for (_, N, K) in w.shapes}))
def test_random_planes_at_every_config_shape(shape):
    N, K = shape
    rng = np.random.default_rng(N * 7 + K)
    t = synth.draw_trits(rng, (N, K), 0.4)
    td = dev(t)
    w = api.pack_exec(td)
    assert np.array_equal(w.cpu().numpy().view(np.uint32), oracle.pack_exec(t)[0])
    assert torch.equal(api.unpack_exec(w, K), td)
    b = api.pack_store(td)
    assert np.array_equal(b.cpu().numpy(), oracle.pack_store(t)[0])
    assert torch.equal(api.unpack_store(b, K), td)


@pytest.mark.parametrize("rows,K", [(1, 1), (3, 4), (5, 7), (2, 16), (7, 333), (4, 2563), (1, 0), (0, 16)])
def test_ragged_store_and_exec(rows, K):
    rng = np.random.default_rng(rows * 1000 + K)
    t = rng.integers(-1, 2, size=(rows, K)).astype(np.int8)
    if rows == 0 or K == 0:
        assert api.pack_store(dev(t)).numel() == 0
        return
    b = api.pack_store(dev(t))
    assert np.array_equal(b.cpu().numpy(), oracle.pack_store(t)[0])
    assert np.array_equal(api.unpack_store(b, K).cpu().numpy(), t)
    if K % 16 == 0:
        w = api.pack_exec(dev(t))
        assert np.array_equal(w.cpu().numpy().view(np.uint32), oracle.pack_exec(t)[0])


def test_invalid_trits_report_and_encode_as_zero():
    rng = np.random.default_rng(1)
    t = rng.integers(-1, 2, size=(9, 64)).astype(np.int8)
    t[2, 3] = 2
    t[8, 63] = -128
    ref_w, bad = oracle.pack_exec(t)
    assert bad == 2
    out = torch.empty((9, 4), dtype=torch.int32, device="cuda")
    assert _lib.load().tern_pack_exec(api._ptr(dev(t)), 9, 64, api._ptr(out), api._stream()) == S["TERN_ERR_BAD_TRIT"]
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref_w)
    ref_b, _ = oracle.pack_store(t)
    outb = torch.empty((9, 13), dtype=torch.uint8, device="cuda")
    assert _lib.load().tern_pack_store(api._ptr(dev(t)), 9, 64, api._ptr(outb), api._stream()) == S["TERN_ERR_BAD_TRIT"]
    assert np.array_equal(outb.cpu().numpy(), ref_b)
    # the next call on a clean input is clean again (status words are per call)
    api.pack_exec(dev(np.zeros((2, 16), np.int8)))


def test_noncanonical_padding_is_reported():
    t = np.zeros((1, 7), np.int8)
    b, _ = oracle.pack_store(t)
    b[0, 1] = b[0, 1] + 9          # third digit of the last byte (a padding digit) from 1 to 2
    ref, bad = oracle.unpack_store(b, 7)
    assert bad == 1
    out = torch.empty((1, 7), dtype=torch.int8, device="cuda")
    assert _lib.load().tern_unpack_store(api._ptr(dev(b)), 1, 7, api._ptr(out), api._stream()) == S["TERN_ERR_BAD_CODE"]
    assert np.array_equal(out.cpu().numpy(), ref)


def test_plane2_survives_roundtrip():
    # the lossy packing the 4B paper excludes (section 9.2) dropped the second plane; here it round-trips
    t = next(synth.draw_workload(synth.WORKLOADS[4], only=["k"]))
    w = api.TernWeight.from_numpy(t.T1, t.s1, t.res_rows, t.T2, t.s2)
    assert torch.equal(api.unpack_exec(w.plane2, t.K).cpu(), torch.from_numpy(t.T2))
    assert torch.equal(w.scale2.cpu(), torch.from_numpy(t.s2))
    api.weight_validate(w)


def test_weight_validate_catches_corruption():
    t = next(synth.draw_workload(synth.WORKLOADS[2], only=["k"]))
    w = api.TernWeight.from_numpy(t.T1, t.s1, t.res_rows, t.T2, t.s2)
    api.weight_validate(w)
    w.plane1.view(-1)[12345] = -1                 # all codes 3
    expect_status(api.weight_validate, w, status="TERN_ERR_BAD_CODE")
    w = api.TernWeight.from_numpy(t.T1, t.s1, t.res_rows, t.T2, t.s2)
    w.res_slot[int(t.res_rows[0])] = 5 if t.r > 6 else -1
    expect_status(api.weight_validate, w, status="TERN_ERR_RESIDUAL")
    w = api.TernWeight.from_numpy(t.T1, t.s1, t.res_rows, t.T2, t.s2)
    w.res_rows[0], w.res_rows[1] = int(t.res_rows[1]), int(t.res_rows[0])
    expect_status(api.weight_validate, w, status="TERN_ERR_RESIDUAL")


# ------------------------------------------------------------------ residual-row metadata
@pytest.mark.parametrize("N", [1, 7, 9, 64, 65, 1000, 4096, 12288])
def test_residual_metadata_bit_exact(N):
    rng = np.random.default_rng(N + 5)
    for frac in (0.0, 0.1, 0.15, 1.0):
        r = int(round(frac * N))
        rows = np.sort(rng.choice(N, size=r, replace=False)).astype(np.int32)
        slot, bm = api.pack_residual(dev(rows), N)
        assert np.array_equal(slot.cpu().numpy(), oracle.slot_map(N, rows))
        assert np.array_equal(bm.cpu().numpy(), oracle.row_bitmap(N, rows))
        rows2, slot2 = api.unpack_residual(bm, N)
        assert np.array_equal(rows2.cpu().numpy(), rows)
        assert np.array_equal(slot2.cpu().numpy(), oracle.slot_map(N, rows))


def test_residual_metadata_large_n_spans_several_scan_rounds():
    # 8 bytes per thread round trip: 1024 threads x 8 rows per round, so N = 3e5 takes ~37 rounds
    N = 300_001
    rng = np.random.default_rng(3)
    rows = np.sort(rng.choice(N, size=45_000, replace=False)).astype(np.int32)
    slot, bm = api.pack_residual(dev(rows), N)
    assert np.array_equal(bm.cpu().numpy(), oracle.row_bitmap(N, rows))
    rows2, slot2 = api.unpack_residual(bm, N)
    assert np.array_equal(rows2.cpu().numpy(), rows)
    assert np.array_equal(slot2.cpu().numpy(), oracle.slot_map(N, rows))


@pytest.mark.parametrize("bad", [[3, 3], [5, 2], [-1, 4], [2, 10]])
def test_pack_residual_rejects_unsorted_or_out_of_range(bad):
    expect_status(api.pack_residual, dev(np.array(bad, np.int32)), 10, status="TERN_ERR_RESIDUAL")


def test_unpack_residual_flags_bits_past_n_and_small_capacity():
    lib = _lib.load()
    bm = dev(np.array([0b00000101, 0b11000001], np.uint8))     # rows 0, 2, 8 valid; bits 14, 15 past N = 10
    import ctypes
    r = ctypes.c_int64(0)
    rows = torch.full((8,), -7, dtype=torch.int32, device="cuda")
    st = lib.tern_unpack_residual(api._ptr(bm), 10, api._ptr(rows), 8, ctypes.byref(r), None, api._stream())
    assert st == S["TERN_ERR_BAD_CODE"] and r.value == 3
    assert rows.cpu().numpy()[:3].tolist() == [0, 2, 8]
    ok = dev(np.array([0b00000101, 0b00000001], np.uint8))
    st = lib.tern_unpack_residual(api._ptr(ok), 10, api._ptr(rows), 2, ctypes.byref(r), None, api._stream())
    assert st == S["TERN_ERR_WORKSPACE"] and r.value == 3


def test_validate_accepts_a_null_slot_map_without_residual_rows():
    rng = np.random.default_rng(1)
    t = synth.draw_tensor(rng, "t", 64, 256, 1, p_zero=0.4, res_pct=0)
    w = api.TernWeight.from_numpy(t.T1, t.s1, t.res_rows, t.T2, t.s2)
    c = w.c_struct()
    c.res_slot = None
    import ctypes
    assert _lib.load().tern_weight_validate(ctypes.byref(c), api._stream()) == 0
