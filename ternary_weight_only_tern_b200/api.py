"""Torch-tensor front end of libtern.so: checks dtypes, devices and contiguity, allocates the
outputs with PyTorch, and passes raw pointers and the current CUDA stream to the C ABI.
No arithmetic of the method happens here; every step runs in the library's kernels."""

from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _lib

GROUP = 128


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(device: torch.device | None = None) -> ctypes.c_void_p:
    """The current CUDA stream of `device` (torch's raw accessor where it exists: it is read on
    every call, and the stream object costs microseconds to build)."""
    if _raw_stream is not None and device is not None and device.index is not None:
        return ctypes.c_void_p(_raw_stream(device.index))
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need(t: torch.Tensor, dtype, name: str, ndim: int = 2):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _ptr(t: torch.Tensor | None):
    return ctypes.c_void_p(t.data_ptr() if t is not None and t.numel() else None)


# ------------------------------------------------------------------------------ packing

def pack_exec(trits: torch.Tensor) -> torch.Tensor:
    """int8 [rows, K] -> exec plane as int32 [rows, K/16] (uint32 bit patterns)."""
    _need(trits, torch.int8, "trits")
    rows, K = trits.shape
    out = torch.empty((rows, K // 16), dtype=torch.int32, device=trits.device)
    _lib.check("tern_pack_exec", _lib.load().tern_pack_exec(_ptr(trits), rows, K, _ptr(out), _stream(trits.device)))
    return out


def unpack_exec(words: torch.Tensor, K: int) -> torch.Tensor:
    _need(words, torch.int32, "words")
    rows = words.shape[0]
    if words.shape[1] * 16 != K:
        raise ValueError("words must hold K/16 words per row")
    out = torch.empty((rows, K), dtype=torch.int8, device=words.device)
    _lib.check("tern_unpack_exec", _lib.load().tern_unpack_exec(_ptr(words), rows, K, _ptr(out), _stream(words.device)))
    return out


def pack_store(trits: torch.Tensor) -> torch.Tensor:
    """int8 [rows, K] -> base-3 store plane uint8 [rows, ceil(K/5)]."""
    _need(trits, torch.int8, "trits")
    rows, K = trits.shape
    out = torch.empty((rows, -(-K // 5)), dtype=torch.uint8, device=trits.device)
    _lib.check("tern_pack_store", _lib.load().tern_pack_store(_ptr(trits), rows, K, _ptr(out), _stream(trits.device)))
    return out


def unpack_store(data: torch.Tensor, K: int) -> torch.Tensor:
    _need(data, torch.uint8, "data")
    rows = data.shape[0]
    if data.shape[1] != -(-K // 5):
        raise ValueError("data must hold ceil(K/5) bytes per row")
    out = torch.empty((rows, K), dtype=torch.int8, device=data.device)
    _lib.check("tern_unpack_store", _lib.load().tern_unpack_store(_ptr(data), rows, K, _ptr(out), _stream(data.device)))
    return out


def pack_residual(res_rows: torch.Tensor, N: int, bitmap: bool = True):
    """Sorted residual rows int32 [r] -> (slot map int32 [N], row bitmap uint8 [ceil(N/8)] or None)
    by tern_pack_residual."""
    _need(res_rows, torch.int32, "res_rows", ndim=1)
    dev = res_rows.device
    slot = torch.empty(N, dtype=torch.int32, device=dev)
    bm = torch.empty(-(-N // 8), dtype=torch.uint8, device=dev) if bitmap else None
    _lib.check("tern_pack_residual", _lib.load().tern_pack_residual(
        _ptr(res_rows), int(res_rows.numel()), N, _ptr(slot), _ptr(bm), _stream(dev)))
    return slot, bm


def unpack_residual(bitmap: torch.Tensor, N: int):
    """Row bitmap uint8 [ceil(N/8)] -> (residual rows int32 [r], slot map int32 [N]) by
    tern_unpack_residual (two calls: the count, then the rows)."""
    _need(bitmap, torch.uint8, "bitmap", ndim=1)
    if bitmap.numel() != -(-N // 8):
        raise ValueError("bitmap must hold ceil(N/8) bytes")
    dev = bitmap.device
    lib = _lib.load()
    r = ctypes.c_int64(0)
    _lib.check("tern_unpack_residual", lib.tern_unpack_residual(_ptr(bitmap), N, None, 0, ctypes.byref(r), None,
                                                                _stream(dev)))
    rows = torch.empty(max(1, r.value), dtype=torch.int32, device=dev)
    slot = torch.empty(N, dtype=torch.int32, device=dev)
    _lib.check("tern_unpack_residual", lib.tern_unpack_residual(_ptr(bitmap), N, _ptr(rows), rows.numel(),
                                                                ctypes.byref(r), _ptr(slot), _stream(dev)))
    return rows[: r.value], slot


@dataclass
class ElemPlane:
    """An element-level second plane in its listed form (tern_pack_elem): the nonzero trits of
    T2e, one byte each, with per-(group, row) counts and per-(group, 64-row block) bases."""
    N: int
    K: int
    ecount: torch.Tensor     # uint8 [K/128, N]
    ebase: torch.Tensor      # int32 [K/128 * ceil(N/64) + 1]
    eidx: torch.Tensor       # uint8 [nnz2 rounded up to 16]
    nnz2: int


def pack_elem(T2e: torch.Tensor) -> ElemPlane:
    """int8 T2e [N, K] -> its listed form (two calls: the count, then the fill)."""
    _need(T2e, torch.int8, "T2e")
    N, K = T2e.shape
    if K % GROUP:
        raise ValueError("K must be a multiple of 128")
    dev = T2e.device
    ecount = torch.empty((K // GROUP, N), dtype=torch.uint8, device=dev)
    ebase = torch.empty(K // GROUP * (-(-N // 64)) + 1, dtype=torch.int32, device=dev)
    nnz = ctypes.c_int64(0)
    lib = _lib.load()
    _lib.check("tern_pack_elem", lib.tern_pack_elem(_ptr(T2e), N, K, _ptr(ecount), _ptr(ebase), None, 0,
                                                    ctypes.byref(nnz), _stream(dev)))
    eidx = torch.empty(max(16, -(-nnz.value // 16) * 16), dtype=torch.uint8, device=dev)
    _lib.check("tern_pack_elem", lib.tern_pack_elem(_ptr(T2e), N, K, _ptr(ecount), _ptr(ebase), _ptr(eidx),
                                                    eidx.numel(), ctypes.byref(nnz), _stream(dev)))
    return ElemPlane(N, K, ecount, ebase, eidx, int(nnz.value))


def unpack_elem(e: ElemPlane) -> torch.Tensor:
    out = torch.empty((e.N, e.K), dtype=torch.int8, device=e.ecount.device)
    _lib.check("tern_unpack_elem", _lib.load().tern_unpack_elem(_ptr(e.ecount), _ptr(e.ebase), _ptr(e.eidx), e.nnz2,
                                                                e.N, e.K, _ptr(out), _stream(out.device)))
    return out


# ------------------------------------------------------------------------------ weights

@dataclass
class TernWeight:
    """A ternarized weight W [N, K] in execution form, on one CUDA device."""
    N: int
    K: int
    plane1: torch.Tensor     # int32 [N, K/16]
    scale1: torch.Tensor     # float16 [N, K/128]
    res_rows: torch.Tensor   # int32 [r]
    res_slot: torch.Tensor   # int32 [N]
    plane2: torch.Tensor     # int32 [r, K/16]
    scale2: torch.Tensor     # float16 [r, K/128]
    static: bool = False     # weights not written by queued work: tern_linear may prefetch them early
    mu: torch.Tensor | None = None   # float16 [N, K/128] per-group offset: W = mu + s1 T1 (+ s2 T2)
    elem: ElemPlane | None = None    # element-level second plane (then r == 0)
    escale: torch.Tensor | None = None   # float16 [N, K/128] its scales s2e
    res_hint: torch.Tensor | None = None  # host int16 [ceil(N/16)] residual rows per strip (a launch hint)

    @property
    def r(self) -> int:
        return int(self.res_rows.numel())

    @property
    def device(self) -> torch.device:
        return self.plane1.device

    def __setattr__(self, name, value):
        # a changed field drops the cached C descriptor and workspace sizes
        object.__setattr__(self, name, value)
        if name not in ("_c", "_ws"):
            object.__setattr__(self, "_c", None)
            object.__setattr__(self, "_ws", None)

    def c_struct(self) -> _lib.TernWeightC:
        c = getattr(self, "_c", None)
        if c is None:
            c = _lib.TernWeightC(
                self.N, self.K, GROUP, self.plane1.data_ptr(), self.scale1.data_ptr(), self.r,
                self.res_rows.data_ptr() if self.r else None, self.res_slot.data_ptr(),
                self.plane2.data_ptr() if self.r else None, self.scale2.data_ptr() if self.r else None,
                _lib.WEIGHT_STATIC if self.static else 0, self.mu.data_ptr() if self.mu is not None else None,
                *self._elem_fields(), self.res_hint.data_ptr() if self.res_hint is not None else None)
            object.__setattr__(self, "_c", c)
        return c

    def _elem_fields(self):
        e = self.elem
        if e is None:
            return (None, None, None, None, 0)
        return (e.ecount.data_ptr(), e.ebase.data_ptr(), e.eidx.data_ptr(), self.escale.data_ptr(), e.nnz2)

    def nbytes(self) -> int:
        """Bytes the decode kernels stream per call: the planes, their scales, the slot map, the
        offset and the element plane's counts, bases, listed trits and scales."""
        ts = (self.plane1, self.scale1, self.plane2, self.scale2, self.res_slot)
        if self.mu is not None:
            ts = ts + (self.mu,)
        n = sum(t.numel() * t.element_size() for t in ts)
        if self.elem is not None:
            e = self.elem
            n += e.ecount.numel() + 4 * e.ebase.numel() + e.nnz2 + 2 * self.escale.numel()
        return n

    @classmethod
    def from_trits(cls, T1: torch.Tensor, s1: torch.Tensor, res_rows: torch.Tensor | None = None,
                   T2: torch.Tensor | None = None, s2: torch.Tensor | None = None,
                   mu: torch.Tensor | None = None, T2e: torch.Tensor | None = None,
                   s2e: torch.Tensor | None = None) -> "TernWeight":
        """Packs int8 planes on the device (tern_pack_exec) and builds the residual-row slot map;
        mu, if given, is the per-group offset [N, K/128]; T2e and s2e, if given, an element-level
        second plane (tern_pack_elem) and its scales, in place of residual rows."""
        _need(T1, torch.int8, "T1")
        _need(s1, torch.float16, "s1")
        N, K = T1.shape
        dev = T1.device
        if res_rows is None or res_rows.numel() == 0:
            res_rows = torch.zeros(0, dtype=torch.int32, device=dev)
            T2 = torch.zeros((0, K), dtype=torch.int8, device=dev)
            s2 = torch.zeros((0, K // GROUP), dtype=torch.float16, device=dev)
        res_rows = res_rows.to(device=dev, dtype=torch.int32).contiguous()
        r = int(res_rows.numel())
        slot, _ = pack_residual(res_rows, N, bitmap=False)
        plane2 = pack_exec(T2) if r else torch.zeros((0, K // 16), dtype=torch.int32, device=dev)
        if mu is not None:
            _need(mu, torch.float16, "mu")
            if tuple(mu.shape) != (N, K // GROUP):
                raise ValueError(f"mu must have shape {(N, K // GROUP)}")
            mu = mu.to(dev).contiguous()
        elem = None
        if T2e is not None:
            if r:
                raise ValueError("a weight carries residual rows or an element plane, not both")
            if tuple(T2e.shape) != (N, K):
                raise ValueError(f"T2e must have shape {(N, K)}")
            _need(s2e, torch.float16, "s2e")
            if tuple(s2e.shape) != (N, K // GROUP):
                raise ValueError(f"s2e must have shape {(N, K // GROUP)}")
            elem = pack_elem(T2e.to(dev).contiguous())
            s2e = s2e.to(dev).contiguous()
        # residual rows per 16-row strip (tern_residual_strip_counts), kept on the host for the decode
        # launches' CTA split
        hint = None
        if r:
            rows_h = res_rows.cpu()
            hint = torch.zeros((N + 15) // 16, dtype=torch.int16)
            _lib.check("tern_residual_strip_counts", _lib.load().tern_residual_strip_counts(
                _ptr(rows_h), r, N, _ptr(hint)))
        return cls(N, K, pack_exec(T1), s1.contiguous(), res_rows, slot, plane2,
                   s2.contiguous() if r else torch.zeros((0, K // GROUP), dtype=torch.float16, device=dev), mu=mu,
                   elem=elem, escale=s2e if elem is not None else None, res_hint=hint)

    @classmethod
    def from_numpy(cls, T1, s1, res_rows, T2, s2, device="cuda", mu=None, T2e=None, s2e=None) -> "TernWeight":
        t = lambda a, dt: torch.from_numpy(a).to(device=device, dtype=dt).contiguous()  # noqa: E731
        return cls.from_trits(t(T1, torch.int8), t(s1, torch.float16), t(res_rows, torch.int32),
                              t(T2, torch.int8), t(s2, torch.float16),
                              mu=t(mu, torch.float16) if mu is not None else None,
                              T2e=t(T2e, torch.int8) if T2e is not None else None,
                              s2e=t(s2e, torch.float16) if s2e is not None else None)


def weight_validate(w: TernWeight) -> None:
    _lib.check("tern_weight_validate", _lib.load().tern_weight_validate(ctypes.byref(w.c_struct()),
                                                                         _stream(w.device)))


# ------------------------------------------------------------------------------ linear

def workspace_bytes(w: TernWeight, M: int) -> int:
    """tern_linear_workspace_bytes, remembered per weight and M."""
    cache = getattr(w, "_ws", None)
    if cache is None:
        cache = {}
        object.__setattr__(w, "_ws", cache)
    n = cache.get(M)
    if n is None:
        n = cache[M] = int(_lib.load().tern_linear_workspace_bytes(ctypes.byref(w.c_struct()), M))
    return n


def linear(x: torch.Tensor, w: TernWeight, out: torch.Tensor | None = None,
           workspace: torch.Tensor | None = None, prefetch: TernWeight | None = None) -> torch.Tensor:
    """y [M, N] = x [M, K] . W^T (fp16 in, fp32 accumulation, fp16 out).

    prefetch: the weight of the next call, whose planes and scales the same launch starts
    bringing into L2 (a cache hint; the result does not depend on it)."""
    _need(x, torch.float16, "x")
    M, K = x.shape
    if K != w.K:
        raise ValueError(f"x has K={K}, weight has K={w.K}")
    if out is None:
        out = torch.empty((M, w.N), dtype=torch.float16, device=x.device)
    else:
        _need(out, torch.float16, "out")
        if tuple(out.shape) != (M, w.N):
            raise ValueError(f"out must have shape {(M, w.N)}, got {tuple(out.shape)}")
    need = workspace_bytes(w, M)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if prefetch is None:
        _lib.check("tern_linear", _lib.load().tern_linear(
            ctypes.byref(w.c_struct()), _ptr(x), M, _ptr(out), _ptr(workspace), ws_bytes, _stream(x.device)))
    else:
        _lib.check("tern_linear_with_prefetch", _lib.load().tern_linear_with_prefetch(
            ctypes.byref(w.c_struct()), _ptr(x), M, _ptr(out), _ptr(workspace), ws_bytes,
            ctypes.byref(prefetch.c_struct()), _stream(x.device)))
    return out


def _weight_array(ws: list):
    """The C array of the weights' descriptor addresses, kept on the first weight per group (the
    key holds the descriptors' addresses, which stay valid while the entry holds them)."""
    structs = [w.c_struct() for w in ws]
    key = tuple(ctypes.addressof(c) for c in structs)
    cache = getattr(ws[0], "_groups", None)
    if cache is None:
        cache = {}
        object.__setattr__(ws[0], "_groups", cache)
    hit = cache.get(key)
    if hit is None:
        hit = cache[key] = ((ctypes.c_void_p * len(ws))(*key), structs)
    return hit[0]


def decode_ranges(ws: list, M: int):
    """(ranges, strips per block, stages per block) of the persistent decode launch that
    linear_group(x [M, K], ws) makes, by tern_decode_ranges: CTA b takes strips
    [ranges[b], ranges[b + 1]); ([], 0, 0) when the call runs no persistent decode kernel."""
    cap = 1024
    arr = (ctypes.c_int32 * (cap + 1))()
    n, sb, ns = ctypes.c_int32(0), ctypes.c_int32(0), ctypes.c_int32(0)
    _lib.check("tern_decode_ranges", _lib.load().tern_decode_ranges(
        _weight_array(ws), len(ws), M, arr, cap, ctypes.byref(n), ctypes.byref(sb), ctypes.byref(ns)))
    return (list(arr[: n.value + 1]) if n.value else []), sb.value, ns.value


def linear_group(x: torch.Tensor, ws: list, outs: list | None = None, workspace: torch.Tensor | None = None,
                 prefetch: list | None = None) -> list:
    """[x . W_i^T for W_i in ws]: weights that share the input x (same K), one decode launch for
    M <= 16. prefetch: the weights of the next call (a cache hint)."""
    _need(x, torch.float16, "x")
    M, K = x.shape
    if not 1 <= len(ws) <= 4 or any(w.K != K for w in ws):
        raise ValueError("linear_group takes 1 to 4 weights with the input's K")
    if outs is None:
        outs = [torch.empty((M, w.N), dtype=torch.float16, device=x.device) for w in ws]
    for o, w in zip(outs, ws):
        _need(o, torch.float16, "out")
        if tuple(o.shape) != (M, w.N):
            raise ValueError(f"out must have shape {(M, w.N)}, got {tuple(o.shape)}")
    need = max(workspace_bytes(w, M) for w in ws)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    warr = _weight_array(ws)
    yarr = (ctypes.c_void_p * len(ws))(*[o.data_ptr() for o in outs])
    pf = list(prefetch or [])
    pstructs = [w.c_struct() for w in pf]
    parr = (ctypes.c_void_p * max(1, len(pf)))(*[ctypes.addressof(c) for c in pstructs])
    _lib.check("tern_linear_group", _lib.load().tern_linear_group(
        warr, len(ws), _ptr(x), M, yarr, _ptr(workspace), ws_bytes, parr if pf else None, len(pf),
        _stream(x.device)))
    return outs


def fit(W: torch.Tensor, res_rows: torch.Tensor | None = None, offset: bool = True, iters: int = 15):
    """Dense fp16 W [N, K] -> (T1 int8 [N, K], s1 [N, K/128], mu [N, K/128] or None, T2 int8 [r, K],
    s2 [r, K/128]) by tern_fit, the second plane on the sorted rows res_rows."""
    _need(W, torch.float16, "W")
    N, K = W.shape
    dev = W.device
    G = K // GROUP
    if res_rows is None or res_rows.numel() == 0:
        res_rows = torch.zeros(0, dtype=torch.int32, device=dev)
    res_rows = res_rows.to(device=dev, dtype=torch.int32).contiguous()
    r = int(res_rows.numel())
    slot, _ = pack_residual(res_rows, N, bitmap=False)
    T1 = torch.empty((N, K), dtype=torch.int8, device=dev)
    s1 = torch.empty((N, G), dtype=torch.float16, device=dev)
    mu = torch.empty((N, G), dtype=torch.float16, device=dev) if offset else None
    T2 = torch.empty((r, K), dtype=torch.int8, device=dev)
    s2 = torch.empty((r, G), dtype=torch.float16, device=dev)
    _lib.check("tern_fit", _lib.load().tern_fit(_ptr(W), N, K, _ptr(slot) if r else None, r, int(offset), iters,
                                                _ptr(T1), _ptr(s1), _ptr(mu), _ptr(T2), _ptr(s2), _stream(dev)))
    return T1, s1, mu, T2, s2


def rotate(x: torch.Tensor, R: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """x [M, K] . blockdiag(R[0], ..., R[K/128 - 1]) with R fp16 [K/128, 128, 128] (tern_rotate)."""
    _need(x, torch.float16, "x")
    _need(R, torch.float16, "R", ndim=3)
    M, K = x.shape
    if tuple(R.shape) != (K // GROUP, GROUP, GROUP) or K % GROUP:
        raise ValueError(f"R must have shape {(K // GROUP, GROUP, GROUP)}")
    if out is None:
        out = torch.empty_like(x)
    else:
        _need(out, torch.float16, "out")
        if tuple(out.shape) != (M, K):
            raise ValueError(f"out must have shape {(M, K)}")
    _lib.check("tern_rotate", _lib.load().tern_rotate(_ptr(x), M, K, _ptr(R), _ptr(out), _stream(x.device)))
    return out


# ------------------------------------------------------------------------------ bits

def bits_elem(N: int, K: int, masked: int, nnz2: int, group: int = GROUP, offset: bool = False) -> dict:
    rep = _lib.TernBitsReport()
    _lib.check("tern_bits_elem", _lib.load().tern_bits_elem(N, K, masked, nnz2, group, int(offset),
                                                            ctypes.byref(rep)))
    return {f: getattr(rep, f) for f, _ in rep._fields_}


def bits(N: int, K: int, r: int, group: int = GROUP, offset: bool = False) -> dict:
    rep = _lib.TernBitsReport()
    fn = "tern_bits_offset" if offset else "tern_bits"
    _lib.check(fn, getattr(_lib.load(), fn)(N, K, r, group, ctypes.byref(rep)))
    return {f: getattr(rep, f) for f, _ in rep._fields_}
