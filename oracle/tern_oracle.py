"""CPU oracle for the weight-only ternary linear layer (W1.58A16).

TEST INFRASTRUCTURE ONLY. Only the tests, the package entry's smoke check and the
bench's CPU-baseline leg may import this module. The CUDA library never calls it,
and it shares no code, table or constant generator with the CUDA sources.

Everything here is the plain definition, written out in float64 (or exact
integers) with numpy, with no blocking, fusion or reordering:

* The representation (what a ternarized weight is):
  - "Post-Training Ternarization of Qwen3-4B: Capability, Effective Bit Budget,
    Storage Compression, and Deployment" (arXiv 2609.01962v1), section 4.3
    (order-2 residual ternarization: ternary planes, each with its own scales),
    section 4.4 (a salience-selected subset of weights gets a second plane),
    section 4.5 (block and group size 128) and section 3.1 (weight-only: the
    activations stay 16-bit).
  - the Qwen3-8B scale-up paper (arXiv 2609.09240), its representation
    paragraph: one ternary plane for most weights, a second plane on a
    salience-selected subset, with per-group scales.
  The row form of the subset (whole output rows carry the second plane) is the
  reading this library builds; the CUDA path follows the same reading.
* The per-group offset (an optional extension of the layer): E2M-ATQ represents
  a group's values as {mu - a, mu, mu + a} around an asymmetric offset (4B
  paper, section 4.3), and the packed format persists scales and offsets (4B
  paper, section 9.1; 8B paper, its footnote on per-group offsets/scales). Read
  here as one fp16 offset per (row, 128-wide group), added once to the
  reconstructed weight: W = mu + s1 T1 (+ s2 T2 on the residual rows).
* The element-level second plane (an optional extension of the layer): the
  8B paper's representation paragraph and the 4B paper's section 4.4 give the
  second plane to the weights of the two most salient of four disjoint
  element masks (3.6 % of a recorded projection's weights). Read here as a
  second ternary plane T2e over all of W that is zero outside the masks, with
  its own fp16 scale per (row, group): W += s2e[n, k // 128] * T2e[n, k]. It
  is kept as a list of its nonzero trits per (row, group), defined below by
  its closed form (the layout is this library's own).
* The activation-side rotation (an optional step before the layer): the pages'
  KOTMS rotation puts the weights into a ternary-friendly basis with structured
  orthogonal matrices, and inference applies the equivalent rotation to the
  activations before the quantized linear operation (4B paper, section 4.2;
  the measured path adds that activation-side matrix operation, section 10.1).
  The structure is not on the pages; read here as block-diagonal with one
  128 x 128 block per 128-wide K group (the method's group size):
  x' = x . blockdiag(R_0, ..., R_{G-1}), so that x' . (W R)^T = x . W^T for
  orthogonal R.
* The ternarization fit (an optional step before packing): E2M-ATQ fits an
  asymmetric offset and two ternary planes with scales, then refines them for 15
  iterations with the ternary supports held fixed (4B paper, section 4.3). Its
  equations are not on the pages. Read here, per (row, 128-wide group), as:
  the offset is the group mean; each plane is the sign of the residual where
  its magnitude exceeds 0.7 times the residual's mean magnitude (the threshold
  rule of ternary weight networks), with the mean magnitude over that support
  as its scale; the second plane fits the first plane's residual, on the rows
  that carry one; the refinement updates the offset, then a1, then a2, each to
  its least-squares value with the others and both planes fixed. Every sum runs
  in float64 over the group's 128 entries in index order, and each of the four
  operations is rounded on its own (no fused multiply-add), so the CUDA path
  reaches every decision with the same numbers.
* The product: with weights in {-1, 0, +1} the matrix product reduces to adding
  and subtracting activations ("Can Ternary LLMs Hit 1.58 Bits per Weight?",
  promptzone, section "What It Is and How It Works"); the oracle computes it
  as the dense float64 product of x with the dequantised W (library matmul),
  which equals that sum of signed activations exactly up to rounding order.
* Packing: the pages say only that the packed format persists the ternary
  planes and scales losslessly (4B paper, section 9.1, Table 6; 8B paper,
  storage discussion). The two byte layouts (2-bit execution codes and
  base-3 storage bytes) are this library's own and are defined here by their
  closed forms.
* Bit accounting: the 4B paper, sections 3.2, 4.4 and 7.1 (1.641 effective
  bits per weight against the ideal log2 3 = 1.585), and the 8B paper's
  effective-bits equation (lost in extraction; read here as log2 3 per plane
  symbol, with a fraction f2 of weights carrying a second plane).

Every function was pinned against something other than itself by the
``-m "not gpu"`` tests (brute force with exact rationals, closed forms,
Python's own base conversion, page figures).
"""

from __future__ import annotations

import math

import numpy as np

GROUP = 128          # scales are per (row, 128 consecutive K columns); 4B paper section 4.5
CODES_PER_WORD = 16  # 2-bit execution codes per uint32 word
TRITS_PER_BYTE = 5   # base-3 storage: 3**5 = 243 <= 256
HEADER_BITS = 512    # a 64-byte container header, counted by the bit accounting


# --------------------------------------------------------------------------------------
# 2-bit execution plane: code c = t + 1 in {0, 1, 2}; 16 codes per uint32 word,
# trit k of a row at bits 2*(k % 16) of word k // 16 (least significant first).
# --------------------------------------------------------------------------------------

def pack_exec(trits: np.ndarray) -> tuple[np.ndarray, int]:
    """int8 trits [rows, K] -> uint32 words [rows, K/16].

    Returns (words, n_invalid). An entry outside {-1, 0, +1} is counted as
    invalid and encoded as the code of 0, which is what the CUDA path writes
    too.
    """
    t = np.asarray(trits, dtype=np.int8)
    rows, K = t.shape
    if K % CODES_PER_WORD:
        raise ValueError("K must be a multiple of 16")
    invalid = (t < -1) | (t > 1)
    codes = np.where(invalid, 1, t.astype(np.int64) + 1).astype(np.uint32)
    codes = codes.reshape(rows, K // CODES_PER_WORD, CODES_PER_WORD)
    words = np.zeros((rows, K // CODES_PER_WORD), dtype=np.uint32)
    for i in range(CODES_PER_WORD):
        words |= codes[:, :, i] << np.uint32(2 * i)
    return words, int(invalid.sum())


def unpack_exec(words: np.ndarray, K: int) -> tuple[np.ndarray, int]:
    """uint32 words [rows, K/16] -> int8 trits [rows, K].

    Code 3 has no trit: it is counted as invalid and decoded as 0.
    """
    w = np.asarray(words, dtype=np.uint32)
    rows = w.shape[0]
    if w.shape[1] * CODES_PER_WORD != K:
        raise ValueError("words do not hold K codes per row")
    shifts = (2 * np.arange(CODES_PER_WORD, dtype=np.uint32))
    codes = (w[:, :, None] >> shifts[None, None, :]) & np.uint32(3)
    invalid = codes == 3
    t = np.where(invalid, 0, codes.astype(np.int64) - 1).astype(np.int8)
    return t.reshape(rows, K), int(invalid.sum())


# --------------------------------------------------------------------------------------
# Base-3 storage plane: byte j of a row = sum_{i<5} (t[5j+i] + 1) * 3**i; a row holds
# ceil(K/5) bytes; positions past K in the last byte hold trit 0 (digit 1).
# --------------------------------------------------------------------------------------

def store_row_bytes(K: int) -> int:
    return -(-K // TRITS_PER_BYTE)


def pack_store(trits: np.ndarray) -> tuple[np.ndarray, int]:
    """int8 trits [rows, K] -> uint8 bytes [rows, ceil(K/5)]; returns (bytes, n_invalid)."""
    t = np.asarray(trits, dtype=np.int8)
    rows, K = t.shape
    nb = store_row_bytes(K)
    invalid = (t < -1) | (t > 1)
    digits = np.ones((rows, nb * TRITS_PER_BYTE), dtype=np.int64)   # pad digit 1 = trit 0
    digits[:, :K] = np.where(invalid, 1, t.astype(np.int64) + 1)
    digits = digits.reshape(rows, nb, TRITS_PER_BYTE)
    value = np.zeros((rows, nb), dtype=np.int64)
    for i in range(TRITS_PER_BYTE):
        value += digits[:, :, i] * (3 ** i)
    return value.astype(np.uint8), int(invalid.sum())


def unpack_store(data: np.ndarray, K: int) -> tuple[np.ndarray, int]:
    """uint8 bytes [rows, ceil(K/5)] -> int8 trits [rows, K].

    A byte >= 243 is not a base-3 number of five digits: it is counted invalid and
    all five of its trits decode as 0. A padding digit (position >= K) other than
    1 is a non-canonical encoding and is counted invalid too (the decoded trits
    are unaffected).
    """
    b = np.asarray(data, dtype=np.uint8)
    rows, nb = b.shape
    if nb != store_row_bytes(K):
        raise ValueError("row length does not match K")
    bad_byte = b >= 243
    v = b.astype(np.int64)
    digits = np.empty((rows, nb, TRITS_PER_BYTE), dtype=np.int64)
    for i in range(TRITS_PER_BYTE):
        digits[:, :, i] = v % 3
        v //= 3
    digits[bad_byte] = 1
    flat = digits.reshape(rows, nb * TRITS_PER_BYTE)
    bad_pad = (flat[:, K:] != 1).any(axis=1) & ~bad_byte[:, -1] if nb * TRITS_PER_BYTE > K else np.zeros(rows, bool)
    t = (flat[:, :K] - 1).astype(np.int8)
    return t, int(bad_byte.sum()) + int(bad_pad.sum())


# --------------------------------------------------------------------------------------
# Residual-row metadata
# --------------------------------------------------------------------------------------

def slot_map(N: int, res_rows: np.ndarray) -> np.ndarray:
    """int32 [N]: -1 for a row with one plane, else the row's index in res_rows."""
    slot = np.full(N, -1, dtype=np.int32)
    slot[np.asarray(res_rows, dtype=np.int64)] = np.arange(len(res_rows), dtype=np.int32)
    return slot


def row_bitmap(N: int, res_rows: np.ndarray) -> np.ndarray:
    """uint8 [ceil(N/8)]: bit n % 8 of byte n // 8 is set when row n carries a second plane."""
    bits = np.zeros(N, dtype=np.uint8)
    bits[np.asarray(res_rows, dtype=np.int64)] = 1
    return np.packbits(bits, bitorder="little")


def rows_from_bitmap(N: int, bitmap: np.ndarray) -> np.ndarray:
    """The inverse of row_bitmap: int32 [r], the rows whose bit is set, in increasing order.
    Bits of the last byte past row N - 1 are not rows (they must be 0 in a canonical bitmap)."""
    bits = np.unpackbits(np.asarray(bitmap, dtype=np.uint8), bitorder="little")[:N]
    return np.nonzero(bits)[0].astype(np.int32)


# --------------------------------------------------------------------------------------
# Element-level second plane: the nonzero trits of T2e, one byte each,
#   byte = (k % 128) << 1 | (t < 0),
# ordered by group g, then row n, then k. ecount[g, n] = number of them in (row n, group g);
# ebase[g * NB + b] = index of the first byte of (group g, rows 64 b .. 64 b + 63), with
# NB = ceil(N / 64) and ebase[G * NB] = nnz2.
# --------------------------------------------------------------------------------------
ELEM_BLOCK = 64


def elem_blocks(N: int) -> int:
    return -(-N // ELEM_BLOCK)


def pack_elem(trits: np.ndarray) -> tuple[np.ndarray, np.ndarray, np.ndarray, int]:
    """int8 T2e [N, K] -> (ecount uint8 [G, N], ebase int64 [G*NB + 1], eidx uint8 [nnz2], n_invalid).

    An entry outside {-1, 0, +1} is counted invalid and packed as 0 (not listed)."""
    t = np.asarray(trits, dtype=np.int8)
    N, K = t.shape
    if K % GROUP:
        raise ValueError("K must be a multiple of 128")
    G, NB = K // GROUP, elem_blocks(N)
    invalid = (t < -1) | (t > 1)
    t = np.where(invalid, 0, t)
    ecount = np.zeros((G, N), dtype=np.uint8)
    ebase = np.zeros(G * NB + 1, dtype=np.int64)
    out = []
    for g in range(G):
        for b in range(NB):
            ebase[g * NB + b] = len(out)
            for n in range(b * ELEM_BLOCK, min(N, (b + 1) * ELEM_BLOCK)):
                seg = t[n, g * GROUP:(g + 1) * GROUP]
                ks = np.flatnonzero(seg)                       # ascending k within the group
                ecount[g, n] = len(ks)
                out.extend(int(kk) << 1 | int(seg[kk] < 0) for kk in ks)
    ebase[G * NB] = len(out)
    return ecount, ebase, np.array(out, dtype=np.uint8), int(invalid.sum())


def unpack_elem(ecount, ebase, eidx, N: int, K: int) -> tuple[np.ndarray, int]:
    """(ecount, ebase, eidx) -> int8 T2e [N, K] and the number of inconsistencies found.

    Inconsistent: a count above 128; a block whose counts do not add up to the gap between its
    base and the next; ebase[0] != 0 or ebase[-1] != len(eidx); within (row, group) a k that does
    not increase. The entries that can be placed are placed regardless."""
    ecount = np.asarray(ecount, dtype=np.int64)
    ebase = np.asarray(ebase, dtype=np.int64)
    eidx = np.asarray(eidx, dtype=np.uint8)
    G, NB = K // GROUP, elem_blocks(N)
    T = np.zeros((N, K), dtype=np.int8)
    bad = int(ebase[0] != 0) + int(ebase[G * NB] != len(eidx))
    for g in range(G):
        for b in range(NB):
            i = int(ebase[g * NB + b])
            rows = range(b * ELEM_BLOCK, min(N, (b + 1) * ELEM_BLOCK))
            if sum(int(ecount[g, n]) for n in rows) != int(ebase[g * NB + b + 1]) - i:
                bad += 1
            for n in rows:
                c = int(ecount[g, n])
                if c > GROUP:
                    bad += 1
                last = -1
                for e in range(i, i + c):
                    if 0 <= e < len(eidx):
                        kk, neg = int(eidx[e]) >> 1, int(eidx[e]) & 1
                        if kk <= last:
                            bad += 1
                        last = kk
                        T[n, g * GROUP + kk] = -1 if neg else 1
                i += c
    return T, bad


# --------------------------------------------------------------------------------------
# Dequantisation and the linear layer
# --------------------------------------------------------------------------------------

def dequant(T1, s1, res_rows, T2, s2, rows=None, mu=None, elem=None) -> np.ndarray:
    """Dense float64 W [N, K] (or the listed rows of it).

    W[n, k] = mu[n, k // 128]  (when an offset is given)
              + s1[n, k // 128] * T1[n, k]
              + [n in R] * s2[rho(n), k // 128] * T2[rho(n), k]
              + s2e[n, k // 128] * T2e[n, k]  (when an element plane elem = (T2e, s2e) is given),
    rho(n) = position of n in the sorted residual-row list R.
    fp16 -> float64 is exact, so W is exact in float64.
    """
    T1 = np.asarray(T1)
    N, K = T1.shape
    if K % GROUP:
        raise ValueError("K must be a multiple of 128")
    rows = np.arange(N) if rows is None else np.asarray(rows, dtype=np.int64)
    s1_cols = np.repeat(np.asarray(s1, dtype=np.float64)[rows], GROUP, axis=1)   # s1[n, k // 128]
    W = s1_cols * T1[rows].astype(np.float64)
    res_rows = np.asarray(res_rows, dtype=np.int64)
    if len(res_rows):
        rho = slot_map(N, res_rows)[rows]
        has2 = rho >= 0
        if has2.any():
            s2_cols = np.repeat(np.asarray(s2, dtype=np.float64)[rho[has2]], GROUP, axis=1)
            W[has2] += s2_cols * np.asarray(T2)[rho[has2]].astype(np.float64)
    if mu is not None:
        W += np.repeat(np.asarray(mu, dtype=np.float64)[rows], GROUP, axis=1)   # mu[n, k // 128]
    if elem is not None:
        T2e, s2e = elem
        W += np.repeat(np.asarray(s2e, dtype=np.float64)[rows], GROUP, axis=1) * \
            np.asarray(T2e)[rows].astype(np.float64)
    return W


def linear(x, T1, s1, res_rows, T2, s2, cols=None, mu=None, elem=None) -> np.ndarray:
    """y_ref [M, N] (or [M, len(cols)]) = x . W^T in float64 (x fp16 -> float64 is exact)."""
    W = dequant(T1, s1, res_rows, T2, s2, rows=cols, mu=mu, elem=elem)
    return np.asarray(x, dtype=np.float64) @ W.T


def round_fp16(y: np.ndarray) -> np.ndarray:
    """One round-to-nearest-even conversion of float64 values to fp16."""
    return np.asarray(y, dtype=np.float64).astype(np.float16)


def rel_err(y, y_ref) -> float:
    """max |y - y_ref| / max |y_ref|, the parity measure for fp16 outputs."""
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    denom = float(np.max(np.abs(y_ref))) if y_ref.size else 0.0
    num = float(np.max(np.abs(y - y_ref))) if y_ref.size else 0.0
    if denom == 0.0:
        return num
    return num / denom


# --------------------------------------------------------------------------------------
# Bit accounting
# --------------------------------------------------------------------------------------

def bits(N: int, K: int, r: int, group: int = GROUP, offset: bool = False) -> dict:
    """Bits of one ternarized tensor in its three forms.

    info  : log2(3) per plane symbol, (N + r) * K symbols; per weight this is
            log2(3) * (1 + f2) with f2 = r / N, the fraction of weights with a second plane.
    store : base-3 planes (8 * ceil(K/5) bits per plane row) + fp16 scales per plane row and
            group + the residual-row bitmap (whole bytes) + a 64-byte header.
    exec  : 2-bit planes (2 bits per symbol) + fp16 scales + the int32 slot map [N] + header.
    offset: the tensor carries a per-group offset: + 16 bits per (row, group) in both forms.
    """
    if K % group:
        raise ValueError("K must be a multiple of the group size")
    G = K // group
    weights = N * K
    plane_rows = N + r
    plane_trits = plane_rows * K
    store_bits = 8 * plane_rows * store_row_bytes(K) + 16 * plane_rows * G + 8 * (-(-N // 8)) + HEADER_BITS
    exec_bits = 2 * plane_trits + 16 * plane_rows * G + 32 * N + HEADER_BITS
    if offset:
        store_bits += 16 * N * G
        exec_bits += 16 * N * G
    return {
        "weights": weights,
        "plane_trits": plane_trits,
        "store_bits": store_bits,
        "exec_bits": exec_bits,
        "bpw_info": math.log2(3) * plane_trits / weights,
        "bpw_store": store_bits / weights,
        "bpw_exec": exec_bits / weights,
    }


def bits_elem(N: int, K: int, masked: int, nnz2: int, group: int = GROUP, offset: bool = False) -> dict:
    """Bits of a tensor whose second plane is element-level: `masked` weights carry a second
    symbol (f2 = masked / (N K)), `nnz2` of those symbols are nonzero and listed.

    info  : log2(3) per plane symbol, N K + masked symbols (the pages' accounting, log2(3) (1 + f2)).
    store : base-3 main plane + fp16 s1 + the element plane (8 bits per ecount entry [G, N],
            32 per ebase entry [G NB + 1], 8 per listed trit, 16 per s2e entry [N, G]) + header.
    exec  : the same with the 2-bit main plane.
    offset: + 16 bits per (row, group) in both forms."""
    if K % group:
        raise ValueError("K must be a multiple of the group size")
    G = K // group
    weights = N * K
    plane_trits = weights + masked
    elem_bits = 8 * G * N + 32 * (G * elem_blocks(N) + 1) + 8 * nnz2 + 16 * N * G
    store_bits = 8 * N * store_row_bytes(K) + 16 * N * G + elem_bits + HEADER_BITS
    exec_bits = 2 * weights + 16 * N * G + elem_bits + HEADER_BITS
    if offset:
        store_bits += 16 * N * G
        exec_bits += 16 * N * G
    return {
        "weights": weights,
        "plane_trits": plane_trits,
        "store_bits": store_bits,
        "exec_bits": exec_bits,
        "bpw_info": math.log2(3) * plane_trits / weights,
        "bpw_store": store_bits / weights,
        "bpw_exec": exec_bits / weights,
    }


# --------------------------------------------------------------------------------------
# Activation-side rotation: y[:, 128 g + j] = sum_i x[:, 128 g + i] R[g, i, j]
# --------------------------------------------------------------------------------------

def rotate(x, R) -> np.ndarray:
    """x [M, K] (fp16 -> float64) times the block-diagonal matrix with blocks R [K/128, 128, 128]."""
    x = np.asarray(x, dtype=np.float64)
    R = np.asarray(R, dtype=np.float64)
    M, K = x.shape
    G = K // GROUP
    if K % GROUP or R.shape != (G, GROUP, GROUP):
        raise ValueError("R must hold one 128 x 128 block per 128-wide group of K")
    y = np.empty((M, K), dtype=np.float64)
    for g in range(G):
        cols = slice(g * GROUP, (g + 1) * GROUP)
        y[:, cols] = x[:, cols] @ R[g]
    return y


# --------------------------------------------------------------------------------------
# Ternarization fit (per row and 128-wide group; see the module docstring)
# --------------------------------------------------------------------------------------
TWN_RATIO = 0.7


def _seq_sum(a: np.ndarray) -> np.ndarray:
    """Sum over the last axis, in index order, in float64 (not numpy's pairwise order)."""
    acc = np.zeros(a.shape[:-1], dtype=np.float64)
    for k in range(a.shape[-1]):
        acc = acc + a[..., k]
    return acc


def _threshold_plane(r: np.ndarray):
    """Plane and scale of residual r [..., 128]: t = sign(r) where |r| > 0.7 mean|r|; a = mean |r| on it."""
    delta = TWN_RATIO * (_seq_sum(np.abs(r)) / GROUP)
    t = ((r > delta[..., None]).astype(np.int8) - (r < -delta[..., None]).astype(np.int8)).astype(np.int8)
    n = np.count_nonzero(t, axis=-1)
    s = _seq_sum(np.where(t != 0, np.abs(r), 0.0))
    a = np.where(n > 0, s / np.maximum(n, 1), 0.0)
    return t, a, n


def fit_groups(w: np.ndarray, has2: np.ndarray, offset: bool, iters: int):
    """The fit of groups w [..., 128] (float64); has2 [...] marks groups with a second plane.
    Returns (T1, a1, mu, T2, a2) with the scales and the offset in float64."""
    mu = _seq_sum(w) / GROUP if offset else np.zeros(w.shape[:-1])
    r = w - mu[..., None]
    T1, a1, n1 = _threshold_plane(r)
    e = r - a1[..., None] * T1
    T2, a2, n2 = _threshold_plane(e)
    T2[~has2] = 0
    a2[~has2] = 0.0
    n2[~has2] = 0
    for _ in range(iters):
        if offset:
            mu = _seq_sum((w - a1[..., None] * T1) - a2[..., None] * T2) / GROUP
        a1 = np.where(n1 > 0, _seq_sum(((w - mu[..., None]) - a2[..., None] * T2) * T1) / np.maximum(n1, 1), 0.0)
        a2 = np.where(n2 > 0, _seq_sum(((w - mu[..., None]) - a1[..., None] * T1) * T2) / np.maximum(n2, 1), 0.0)
    return T1, a1, mu, T2, a2


def ternarize(W, res_rows=None, offset: bool = True, iters: int = 15):
    """Dense W [N, K] (fp16 -> float64, exact) -> (T1 int8 [N, K], s1 fp16 [N, G], mu fp16 [N, G] or
    None, T2 int8 [r, K], s2 fp16 [r, G]) with the second plane on the sorted rows res_rows; each
    scale and offset is rounded once to fp16."""
    W = np.asarray(W, dtype=np.float16).astype(np.float64)
    N, K = W.shape
    if K % GROUP:
        raise ValueError("K must be a multiple of 128")
    G = K // GROUP
    res_rows = np.zeros(0, np.int64) if res_rows is None else np.asarray(res_rows, dtype=np.int64)
    has2 = np.zeros((N, G), dtype=bool)
    has2[res_rows] = True
    T1, a1, mu, T2, a2 = fit_groups(W.reshape(N, G, GROUP), has2, offset, iters)
    return (T1.reshape(N, K), a1.astype(np.float16), mu.astype(np.float16) if offset else None,
            T2.reshape(N, K)[res_rows], a2[res_rows].astype(np.float16))
