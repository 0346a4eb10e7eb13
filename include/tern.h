/*
 * tern.h -- C ABI of libtern.so: the weight-only ternary linear layer (W1.58A16) on
 * NVIDIA B200 (sm_100a).
 *
 * What is computed (the representation of the ternarized weights):
 *   y[m, n] = sum_g s1[n, g] * sum_{k in g} T1[n, k] * x[m, k]
 *           + [n in R] * sum_g s2[rho(n), g] * sum_{k in g} T2[rho(n), k] * x[m, k]
 *   - T1, T2 hold trits in {-1, 0, +1}; each s is an fp16 scale per (row, 128-wide K group).
 *     "Post-Training Ternarization of Qwen3-4B: Capability, Effective Bit Budget, Storage
 *     Compression, and Deployment" (arXiv 2609.01962v1), section 4.3 (ternary planes with
 *     scales; an order-2 residual plane), section 4.5 (group size 128).
 *   - R is a salience-selected subset that carries the second plane (4B paper, section 4.4;
 *     the Qwen3-8B scale-up paper, arXiv 2609.09240, representation paragraph). This
 *     library takes the subset as whole output rows; rho(n) is n's index in the sorted R.
 *   - Optionally a per-group offset mu (fp16 [N, K/128]) adds sum_g mu[n, g] * sum_{k in g}
 *     x[m, k] to every row, residual or not (see tern_weight.mu).
 *   - Optionally the second plane is element-level instead of row-level: a plane T2e over all
 *     of W, nonzero only on salience-selected weights, with its own fp16 scale per (row,
 *     group), adds sum_g s2e[n, g] * sum_{k in g} T2e[n, k] * x[m, k] (see "element plane"
 *     below).
 *   - x and y stay fp16 (weight-only quantisation, 4B paper section 3.1); the sums are
 *     accumulated in fp32 and rounded to fp16 once.
 *   - With weights in {-1, 0, +1} the product is additions and subtractions of activations
 *     (promptzone, "Can Ternary LLMs Hit 1.58 Bits per Weight?", section "What It Is and
 *     How It Works"); the kernels feed exact +-x or 0 products to fp32 accumulators.
 *
 * Layouts (all row-major, no padding between rows):
 *   exec plane : uint32 [rows, K/16]; trit k of a row is code c = t + 1 in {0,1,2} at
 *                bits 2*(k % 16) of word k/16 (code 3 is invalid).
 *   store plane: uint8 [rows, ceil(K/5)]; byte j = sum_{i<5} (t[5j+i] + 1) * 3^i, the
 *                positions past K in a row's last byte hold trit 0 (digit 1); bytes >= 243
 *                are invalid.
 *   scales     : fp16 (IEEE binary16 bit patterns, tern_half) [rows, K/128].
 *   x, y       : fp16 [M, K] and [M, N].
 *   Persisting the discrete planes and scales (not a floating reconstruction) is what the
 *   pages' lossless packing does (4B paper, section 9.1 and Table 6; 8B paper, storage
 *   discussion); the two byte layouts are this library's own.
 *
 * Conventions:
 *   - Pointers marked "device" point to device memory of the current CUDA device; the
 *     caller owns every buffer. tern_linear allocates nothing: its only scratch is the
 *     caller's workspace.
 *   - Arguments are validated on the host before any launch; on a host-side error nothing
 *     is launched and nothing is written.
 *   - tern_linear is asynchronous on the given stream and can be captured in a CUDA graph.
 *     The pack and unpack calls are synchronous on their stream: they return only after
 *     the stream has drained, so that they can report invalid codes found on the device.
 *   - `stream` is a cudaStream_t (0 = the legacy default stream).
 */
#ifndef TERN_H
#define TERN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t tern_half;               /* IEEE binary16 bit pattern */
typedef struct CUstream_st* tern_stream;  /* the same type as cudaStream_t */

typedef enum {
    TERN_OK = 0,
    TERN_ERR_NULL = 1,       /* a required pointer is NULL */
    TERN_ERR_SHAPE = 2,      /* a size is negative, K is not a multiple of 128 (16 for the exec
                                plane), group != 128, r > N, or a size is too large */
    TERN_ERR_ALIGN = 3,      /* a pointer is not 16-byte aligned */
    TERN_ERR_BAD_TRIT = 4,   /* pack: an input int8 is outside {-1, 0, +1} */
    TERN_ERR_BAD_CODE = 5,   /* unpack / validate: a 2-bit code 3, a byte >= 243, or a
                                non-canonical padding digit */
    TERN_ERR_RESIDUAL = 6,   /* validate: residual rows not strictly increasing, out of range,
                                or inconsistent with the slot map */
    TERN_ERR_WORKSPACE = 7,  /* workspace smaller than tern_linear_workspace_bytes() or NULL */
    TERN_ERR_CUDA = 8,       /* a CUDA runtime call failed (launch error, no device, ...) */
    TERN_ERR_TIMEOUT = 9,    /* a bounded device-side wait ran out (see tern_device_status) */
    TERN_ERR_ELEM = 10,      /* unpack_elem / validate: element-plane counts, bases or order
                                inconsistent */
    TERN_ERR_BOUNDS = 11     /* a TERN_DEBUG build's device-side bounds check failed (the access was
                                skipped; outputs since the last tern_device_status are undefined) */
} tern_status;

/* A ternarized weight W [N, K] in execution form. Every pointer is device memory,
 * caller-owned, 16-byte aligned, except res_per_strip (host memory).                   */
typedef struct {
    int64_t N, K;                /* output and input features; K % 128 == 0            */
    int32_t group;               /* scale group width along K; must be 128             */
    const uint32_t* plane1;      /* [N, K/16]   exec codes of T1                        */
    const tern_half* scale1;     /* [N, K/128]  s1                                      */
    int64_t r;                   /* rows with a second plane, 0 <= r <= N               */
    const int32_t* res_rows;     /* [r] strictly increasing row indices (R); read only by
                                    tern_weight_validate                                 */
    const int32_t* res_slot;     /* [N] -1, or rho(n) for n in R (tern_pack_residual);
                                    may be NULL when r == 0                              */
    const uint32_t* plane2;      /* [r, K/16]   exec codes of T2                        */
    const tern_half* scale2;     /* [r, K/128]  s2                                      */
    uint32_t flags;              /* 0 or TERN_WEIGHT_STATIC                             */
    const tern_half* mu;         /* [N, K/128]  per-group offset, or NULL (none)        */
    /* element plane (NULL ecount = none; needs r == 0), layout below                    */
    const uint8_t* ecount;       /* [K/128, N]  listed trits of (group g, row n)         */
    const int32_t* ebase;        /* [K/128 * ceil(N/64) + 1] first listed trit of each
                                    (group, 64-row block); the last entry is nnz2        */
    const uint8_t* eidx;         /* [nnz2] listed trits, allocated to a multiple of 16 bytes */
    const tern_half* escale;     /* [N, K/128]  s2e                                     */
    int64_t nnz2;                /* number of listed trits                              */
    /* HOST memory, optional (NULL: none): [ceil(N/16)] the number of residual rows among rows
     * 16 j .. 16 j + 15, for each strip j. With it on every weight of a call that has residual
     * rows, the decode launch splits its strips among the CTAs so that their main and residual
     * blocks even out, instead of splitting the strips evenly (a planning hint read on the host
     * during the call: the results do not depend on it).                                 */
    const uint16_t* res_per_strip;
} tern_weight;

/* With an offset the weight is W[n, k] = mu[n, k/128] + s1[n, k/128] T1[n, k]
 * (+ s2[rho(n), k/128] T2[rho(n), k] on the residual rows): E2M-ATQ's values {mu - a, mu,
 * mu + a} around an asymmetric per-group offset ("Post-Training Ternarization of Qwen3-4B",
 * section 4.3; the packed format keeps scales and offsets, section 9.1). Without one
 * (mu == NULL) W = s1 T1 (+ s2 T2).                                                     */

/* Element plane. The pages give a second ternary plane to the weights of the two most salient
 * of four disjoint element masks (3.6 % of a recorded projection's weights: the Qwen3-8B
 * scale-up paper, representation paragraph; "Post-Training Ternarization of Qwen3-4B",
 * section 4.4). Here that plane is T2e [N, K], zero outside the masks, with one fp16 scale per
 * (row, group): W += s2e[n, k/128] T2e[n, k]. It is kept as the list of its nonzero trits,
 * one byte each, (k % 128) << 1 | (t < 0), ordered by group, then row, then k; ecount[g, n] is
 * the number listed for (row n, group g), and ebase[g * ceil(N/64) + b] the index of the first
 * one of rows 64b .. 64b+63 in group g, so that the trits of one group of 64 consecutive rows
 * are contiguous. A row may carry a row-level second plane (r > 0) or an element plane, not
 * both; an element plane may carry an offset. Every pointer 16-byte aligned.             */

/* tern_weight.flags: the planes, scales and slot map are not written by work queued before
 * the call on its stream (model weights). tern_linear may then start reading them while the
 * previous kernel on the stream is still running (programmatic dependent launch); x is
 * always read only after that kernel has finished.                                      */
#define TERN_WEIGHT_STATIC 1u

/* ---------------------------------------------------------------- packing (offline) */

/* int8 trits t [rows, K] (device) -> exec plane out [rows, K/16] (device). K % 16 == 0.
 * An input outside {-1,0,+1} is encoded as the code of 0 and the call returns
 * TERN_ERR_BAD_TRIT (the rest of `out` is written as usual). Synchronous on `stream`. */
tern_status tern_pack_exec(const int8_t* t, int64_t rows, int64_t K, uint32_t* out, tern_stream stream);

/* exec plane p [rows, K/16] (device) -> int8 trits out [rows, K] (device). A code 3 decodes
 * as 0 and the call returns TERN_ERR_BAD_CODE. Synchronous on `stream`.               */
tern_status tern_unpack_exec(const uint32_t* p, int64_t rows, int64_t K, int8_t* out, tern_stream stream);

/* int8 trits t [rows, K] (device) -> store plane out [rows, ceil(K/5)] (device). Any K >= 0.
 * Invalid trits: as for tern_pack_exec. Synchronous on `stream`.                        */
tern_status tern_pack_store(const int8_t* t, int64_t rows, int64_t K, uint8_t* out, tern_stream stream);

/* store plane b [rows, ceil(K/5)] (device) -> int8 trits out [rows, K] (device). A byte
 * >= 243 decodes as five 0 trits; a padding digit other than 1 is non-canonical; both
 * return TERN_ERR_BAD_CODE. Synchronous on `stream`.                                    */
tern_status tern_unpack_store(const uint8_t* b, int64_t rows, int64_t K, int8_t* out, tern_stream stream);

/* int8 T2e [N, K] (device) -> element plane: ecount [K/128, N], ebase [K/128 * ceil(N/64) + 1]
 * and, when eidx is not NULL, the listed trits eidx (device), of which there are *nnz2.
 * K % 128 == 0. Call once with eidx == NULL to learn *nnz2 (ecount and ebase are written),
 * then with eidx of eidx_bytes >= nnz2 rounded up to 16 (the padding is zeroed); a smaller
 * eidx returns TERN_ERR_WORKSPACE and leaves eidx untouched. An input outside {-1,0,+1} is
 * listed as 0 (not at all) and the call returns TERN_ERR_BAD_TRIT. Synchronous on `stream`. */
tern_status tern_pack_elem(const int8_t* t, int64_t N, int64_t K, uint8_t* ecount, int32_t* ebase, uint8_t* eidx,
                           int64_t eidx_bytes, int64_t* nnz2, tern_stream stream);

/* Element plane (device) -> int8 T2e out [N, K] (device). Inconsistent input (a count above
 * 128, a block whose counts do not add up to the gap between its base and the next, ebase[0]
 * != 0 or the last base != nnz2, a k that does not increase within a (row, group)) returns
 * TERN_ERR_ELEM; every trit whose index lies in [0, nnz2) is still placed. Synchronous.   */
tern_status tern_unpack_elem(const uint8_t* ecount, const int32_t* ebase, const uint8_t* eidx, int64_t nnz2,
                             int64_t N, int64_t K, int8_t* out, tern_stream stream);

/* Residual-row metadata. The second plane is carried by a salience-selected subset R of the
 * output rows ("Post-Training Ternarization of Qwen3-4B", section 4.4; the Qwen3-8B scale-up
 * paper, representation paragraph), which this library keeps as whole rows. Its execution form
 * is the slot map res_slot [N] int32 (-1, or rho(n) = n's index in R), which the linear kernels
 * read; its storage form is a row bitmap [ceil(N/8)] uint8 (bit n % 8 of byte n / 8 set for n in
 * R, the bits past row N - 1 zero), the one counted by tern_bits' store_bits.
 *
 * tern_pack_residual: res_rows [r] (device; strictly increasing, in [0, N)) -> res_slot [N]
 * (device, required when N > 0) and, when row_bitmap is not NULL, the bitmap (device). Rows out
 * of range or not strictly increasing return TERN_ERR_RESIDUAL; the outputs are then written
 * but describe no valid weight. int32 pointers 4-byte aligned. Synchronous on `stream`.     */
tern_status tern_pack_residual(const int32_t* res_rows, int64_t r, int64_t N, int32_t* res_slot,
                               uint8_t* row_bitmap, tern_stream stream);

/* tern_residual_strip_counts: res_rows [r] (HOST; strictly increasing, in [0, N)) -> counts
 * [ceil(N/16)] (host): the residual rows among rows 16 j .. 16 j + 15 of each strip j, the
 * tern_weight.res_per_strip hint. Rows out of range or not strictly increasing return
 * TERN_ERR_RESIDUAL (counts then undefined). Host function.                                */
tern_status tern_residual_strip_counts(const int32_t* res_rows, int64_t r, int64_t N, uint16_t* counts);

/* tern_unpack_residual: row bitmap [ceil(N/8)] (device) -> *r = |R| (host), and, when not
 * NULL, res_rows [r] (device, capacity r_cap entries) in increasing order and res_slot [N]
 * (device). Call with res_rows == NULL to learn *r. A bit set past row N - 1 is not a row and
 * returns TERN_ERR_BAD_CODE (the outputs still hold the rows below N); more than r_cap rows
 * return TERN_ERR_WORKSPACE (the first r_cap are written). Synchronous on `stream`.        */
tern_status tern_unpack_residual(const uint8_t* row_bitmap, int64_t N, int32_t* res_rows, int64_t r_cap,
                                 int64_t* r, int32_t* res_slot, tern_stream stream);

/* Checks a weight descriptor's device data: every code of plane1/plane2 is in {0,1,2},
 * res_rows is strictly increasing in [0, N), and res_slot[n] == i exactly when
 * res_rows[i] == n (else -1; a NULL res_slot is accepted when r == 0); an element plane is
 * checked as by tern_unpack_elem.
 * Returns TERN_OK, TERN_ERR_BAD_CODE, TERN_ERR_RESIDUAL or TERN_ERR_ELEM.
 * Synchronous on `stream`. tern_linear does not repeat these checks; it only keeps its
 * own memory accesses in bounds when a slot is out of range.                            */
tern_status tern_weight_validate(const tern_weight* w, tern_stream stream);

/* Dense fp16 W [N, K] (device) -> the ternary form: T1 int8 [N, K], s1 [N, K/128], with
 * offset != 0 mu [N, K/128], and on the rows n with res_slot[n] = j >= 0 (res_slot [N], as
 * tern_weight.res_slot, or NULL when r == 0) T2[j] int8 [K] and s2[j] [K/128]. Per (row, 128-wide
 * group): mu = the group mean (0 without an offset), T1 = sign(w - mu) where |w - mu| exceeds 0.7
 * times its mean, a1 = the mean magnitude on that support, T2 and a2 the same on the residual
 * w - mu - a1 T1, then `iters` rounds of least-squares updates of mu, a1 and a2 in turn with the
 * planes fixed; sums in float64 in index order, each scale and offset rounded once to fp16.
 * This is the fit the pages call E2M-ATQ (an asymmetric offset, two ternary planes with scales,
 * 15 refinement iterations with the supports fixed: "Post-Training Ternarization of Qwen3-4B",
 * section 4.3) in this library's reading of it (the pages give no equations). The outputs feed
 * tern_pack_exec. W, T1 and T2 16-byte aligned; 0 <= iters <= 1000. Asynchronous on `stream`. */
tern_status tern_fit(const tern_half* W, int64_t N, int64_t K, const int32_t* res_slot, int64_t r, int32_t offset,
                     int32_t iters, int8_t* T1, tern_half* s1, tern_half* mu, int8_t* T2, tern_half* s2,
                     tern_stream stream);

/* ---------------------------------------------------------------- the linear layer */

/* Bytes of workspace tern_linear needs for this weight and batch size (0 if none). */
size_t tern_linear_workspace_bytes(const tern_weight* w, int64_t M);

/* y [M, N] = x [M, K] . W^T for the ternary W above (x, y device, fp16, row-major).
 * M <= 16 runs the decode GEMV (split along K over a thread-block cluster); larger M
 * runs the dequantise-into-tcgen05 GEMM. M == 0 is a no-op returning TERN_OK.
 * x and y must not overlap. Asynchronous on `stream`; capturable in a CUDA graph.
 * workspace: device scratch of at least tern_linear_workspace_bytes(w, M) bytes, owned
 * by the caller, not used by another call that runs at the same time.                  */
tern_status tern_linear(const tern_weight* w, const tern_half* x, int64_t M, tern_half* y,
                        void* workspace, size_t workspace_bytes, tern_stream stream);

/* As tern_linear, and in the same launch starts bringing the planes, scales and slot map of
 * `next` into the L2 cache: a decode loop passes the weight of its next call, whose loads then
 * hit the cache while this call's arithmetic runs. A pure cache hint: `next` is read by no
 * result and may be NULL (then this is tern_linear); its pointers must satisfy the rules of
 * tern_weight, and a descriptor that fails them is reported as for `w`. The prefill path
 * (M > 16) ignores it.                                                                  */
tern_status tern_linear_with_prefetch(const tern_weight* w, const tern_half* x, int64_t M, tern_half* y,
                                      void* workspace, size_t workspace_bytes, const tern_weight* next,
                                      tern_stream stream);

/* y[i] [M, N_i] = x [M, K] . W_i^T for n weights that share one input x (1 <= n <= 4, every
 * W_i with the same K, and either all or none with an element plane): the projections of one
 * activation, such as q, k and v, or gate and up.
 * M <= 16 runs them as one decode-GEMV launch (each weight's 64-row blocks are blocks of the
 * same grid), so the per-launch latency is paid once; larger M runs the GEMM once per weight.
 * `next` (n_next <= 4 weights, or NULL) is prefetched into L2 as by tern_linear_with_prefetch.
 * No y[i] may overlap x or another y[j]. The workspace rule of tern_linear holds for each W_i.
 * Asynchronous on `stream`; capturable in a CUDA graph. w, y and next are host arrays of
 * device descriptors and device pointers.                                                  */
tern_status tern_linear_group(const tern_weight* const* w, int32_t n, const tern_half* x, int64_t M,
                              tern_half* const* y, void* workspace, size_t workspace_bytes,
                              const tern_weight* const* next, int32_t n_next, tern_stream stream);

/* The CTA split of the persistent decode launch that tern_linear_group(w, n, x, M, ...) makes
 * (tern_linear: n = 1), for inspection and tests: CTA b walks the 16-row strips
 * [ranges[b], ranges[b + 1]) of the weights' strips in order (weight i's after those of weights
 * 0 .. i-1), in blocks of *strips_per_block strips of *stages_per_block stages (either pointer
 * may be NULL). With res_per_strip on every weight that has residual rows the split is balanced
 * by the blocks each CTA walks, else even. *n_ctas = 0 when that call runs no persistent decode
 * kernel (M > 16, element planes, a 2-8-token launch the cluster kernel takes). ranges holds
 * max_ctas + 1 entries; TERN_ERR_SHAPE when the launch needs more CTAs (its CTA count is the
 * current device's SM count, 148 without a device). Host function: reads the descriptors and
 * res_per_strip, no device memory; the weights' validity rules of tern_linear apply.       */
tern_status tern_decode_ranges(const tern_weight* const* w, int32_t n, int64_t M, int32_t* ranges,
                               int32_t max_ctas, int32_t* n_ctas, int32_t* strips_per_block,
                               int32_t* stages_per_block);

/* ---------------------------------------------------------------- activation rotation */

/* y [M, K] = x [M, K] . blockdiag(R_0, ..., R_{G-1}) (x, y, R device, fp16, row-major): the
 * rotation that inference applies to the activations before the linear layer when the
 * weights were moved into a rotated basis ("Post-Training Ternarization of Qwen3-4B", section
 * 4.2: KOTMS uses structured orthogonal matrices, and the equivalent rotation is applied to the
 * activations; section 10.1). This library reads the structure as block-diagonal with one
 * 128 x 128 block per 128-wide group of K: R is [K/128, 128, 128] with
 * y[m, 128 g + j] = sum_i x[m, 128 g + i] R[g, i, j], fp32 accumulation, one rounding to fp16.
 * K % 128 == 0; x and y must not overlap. Asynchronous on `stream`; capturable in a CUDA graph.
 * The next kernel on the stream may start while this one runs (programmatic dependent launch):
 * tern_linear reads its x only after this kernel has finished.                           */
tern_status tern_rotate(const tern_half* x, int64_t M, int64_t K, const tern_half* R, tern_half* y,
                        tern_stream stream);

/* ---------------------------------------------------------------- bit accounting */

typedef struct {
    uint64_t weights;       /* N*K                                                      */
    uint64_t plane_trits;   /* (N+r)*K symbols in the ternary planes                    */
    uint64_t store_bits;    /* 8*(N+r)*ceil(K/5) + 16*(N+r)*G + 8*ceil(N/8) + 512       */
    uint64_t exec_bits;     /* 2*(N+r)*K + 16*(N+r)*G + 32*N + 512                      */
    double bpw_info;        /* log2(3) * plane_trits / weights = log2(3) * (1 + r/N)    */
    double bpw_store;       /* store_bits / weights                                     */
    double bpw_exec;        /* exec_bits / weights                                      */
} tern_bits_report;

/* Bits per weight of one ternarized tensor: the information rate of its planes (log2 3 per
 * symbol, with a fraction f2 = r/N of weights carrying a second plane), and the exact bit
 * totals of its storage form (base-3 planes, fp16 scales, the residual-row bitmap, a
 * 64-byte header) and of its execution form (2-bit planes, fp16 scales, the int32 slot map,
 * a 64-byte header). 4B paper, sections 3.2, 4.4 and 7.1 (1.641 effective bits against the
 * ideal 1.585); 8B paper, effective-bits equation. Pure host function.                  */
tern_status tern_bits(int64_t N, int64_t K, int64_t r, int32_t group, tern_bits_report* out);

/* As tern_bits for a tensor that also carries a per-group offset: 16 more bits per
 * (row, group) in the storage and the execution forms; the information figure counts plane
 * symbols only and is unchanged.                                                        */
tern_status tern_bits_offset(int64_t N, int64_t K, int64_t r, int32_t group, tern_bits_report* out);

/* Bits of a tensor whose second plane is element-level: `masked` weights carry a second
 * symbol (the information rate is log2(3) (1 + masked / (N K)), the pages' f2 accounting) and
 * nnz2 of them are listed. store and exec add to the main plane and s1 the element plane's
 * bytes: 8 bits per ecount entry, 32 per ebase entry, 8 per listed trit, 16 per s2e entry;
 * offset != 0 adds 16 bits per (row, group). plane_trits = N K + masked. Host only.      */
tern_status tern_bits_elem(int64_t N, int64_t K, int64_t masked, int64_t nnz2, int32_t group, int32_t offset,
                           tern_bits_report* out);

/* Reports, and clears, the current device's sticky status word for asynchronous work: returns
 * TERN_ERR_TIMEOUT if a tern_linear kernel since the last call gave up a bounded device-side
 * wait (its output is then undefined), TERN_ERR_BOUNDS if, in a TERN_DEBUG build, one of its
 * device-side bounds checks failed (that access was skipped; the output is undefined), else
 * TERN_OK. Synchronous on `stream`.                                                       */
tern_status tern_device_status(tern_stream stream);

/* 1 for a TERN_DEBUG build (libtern_debug.so: the decode kernels check their shared- and global-
 * memory indices before each access and report a failure through tern_device_status instead of
 * faulting), 0 for the release build. No counterpart on the pages: a test aid.            */
int tern_debug_build(void);

/* The failure path of the bounded device-side waits, exercised on purpose: one thread waits on
 * a shared-memory barrier that nothing completes, bounded by `cycles` SM clock cycles
 * (1 <= cycles <= 2^32), and then records the timeout in the device's sticky status word as a
 * linear kernel whose wait ran out does; no copy or MMA is in flight meanwhile, and the context
 * stays usable. A following tern_device_status returns TERN_ERR_TIMEOUT and clears the word.
 * For tests of error handling. Asynchronous on `stream`.                                   */
tern_status tern_selftest_timeout(int64_t cycles, tern_stream stream);

/* A static, human-readable name for a status code. */
const char* tern_status_string(tern_status s);

/* The library's version as major*10000 + minor*100 + patch. */
int tern_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TERN_H */
