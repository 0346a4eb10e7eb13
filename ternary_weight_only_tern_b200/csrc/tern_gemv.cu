// Decode GEMV for M <= 16: y[M, N] = x[M, K] . W^T with W on packed 2-bit ternary planes.
//
// What it computes is the representation of "Post-Training Ternarization of Qwen3-4B"
// (arXiv 2609.01962v1), sections 4.3-4.5: one ternary plane T1 with an fp16 scale per
// (row, 128-wide K group), plus a residual plane T2 with its own scales on a subset R of
// rows; activations stay fp16 (section 3.1). With t in {-1, 0, +1} every product t*x is
// exact, so the layer is a signed sum of activations ("Can Ternary LLMs Hit 1.58 Bits per
// Weight?", promptzone, "What It Is and How It Works"), accumulated here in fp32.
//
// Design (B200; memory-bound at 0.266 bytes per weight):
//  * A CTA owns 64 output rows x one K-slice of at most 8 groups. Its first act is to issue
//    2D TMA loads of its whole weight tile (64 rows x 128 bytes of codes per box, 128-byte
//    swizzle), of the residual-plane rows that belong to those 64 rows and of their scales,
//    so the HBM stream starts at once and no later step waits on another global round trip
//    except the read of x.
//  * The K-slices of a 64-row block form a thread-block cluster. Each CTA sends its partial
//    sums to the rank that owns the row as asynchronous stores into that rank's shared memory
//    (st.async, completing on the owner's receive barrier); the owner adds them in rank order
//    (no global partials, no atomics, a deterministic result) and the CTA of cluster rank c
//    writes rows [c*64/S, (c+1)*64/S). No CTA waits for its peers to finish.
//  * Up to 4 weights that share x run as one launch: each weight's 64-row blocks are blocks of
//    the same grid, and a CTA finds its weight from blockIdx.y.
//  * Warps 0-3 each own a 16-row strip of the main plane. Warp 4 owns the residual rows of the
//    block: since R is sorted, they are the contiguous slots [s_lo, s_lo + nres) of the
//    residual plane, taken 16 rows at a time. Their sums join the main rows' sums before the
//    single rounding to fp16.
//  * The signed sums run on the tensor pipe as mma.sync m16n8k16 (fp16 in, fp32 accumulate):
//    A = 16 weight rows x 16 K of decoded trits, B = the activations of up to 8 tokens. The
//    products are exact (+-x or 0), so this is the fp32-accumulated add/subtract of the
//    method, and the decode cost does not grow with M.
//  * Decode is branch-free: one LOP3 turns two 2-bit codes (bits p and p+16 of a word) into
//    an fp16 pair (B_p + c) by writing the code into the mantissa of a power of two B_p; a
//    shift by 6 either way moves the codes of bits 0-3 and 10-15 into mantissa positions,
//    so a word of 16 trits costs 2 shifts and 8 LOP3. Since c = t + 1, the MMA sums
//    (B_p + 1 + t) * x from zero, and C = sum (B_p + 1) * x is subtracted once per group. C is
//    computed once per CTA by the same MMA on the constant pattern B_p + 1 in the same K order
//    and accumulator split (hidden behind the weight loads), so a zero plane cancels bit for
//    bit. The bases are 4, 16 and 64, so the offsets are small and every partial sum is exact
//    on integer inputs. A non-finite activation makes every output of its token non-finite
//    (NaN where the dense product has +-inf).
//  * Options: a per-group offset mu (section 4.3's asymmetric offset) adds mu * X_g, the
//    group sums X_g coming from one more MMA chain on an all-ones pattern; an element-level
//    second plane (section 4.4's salience masks) is staged by warp 4 and summed on the CUDA
//    cores.
//  * The contraction order over K is free, so the MMA's K order follows the packed words
//    (pair j = trits j and j+8 of a word); x is staged in shared memory in that order, with
//    the words of a group arranged so that one MMA step's activation fragments are 128
//    contiguous bytes (no bank conflicts).
//  * Launches use programmatic dependent launch: a kernel may start while the previous one on
//    the stream drains; it reads x (and, unless the weight is flagged static, the weight)
//    only after griddepcontrol.wait, and writes nothing before it.
#include <stdlib.h>

#include <algorithm>
#include <mutex>

#include "tern_device.cuh"

namespace tern {
namespace {

using namespace dev;

constexpr int kMainWarps = 4;
constexpr int kThreads = (kMainWarps + 1) * 32;     // + one warp for the residual rows
constexpr int kRowsPerCta = 16 * kMainWarps;        // 64
constexpr int kChunkGroups = 4;                     // groups per TMA box: 32 words = 128 bytes per row
constexpr int kMaxGpc = 8;                          // groups per K-slice
constexpr int kMaxChunks = kMaxGpc / kChunkGroups;
constexpr int kStrip = 16;
constexpr int kResStrips = 2;                       // residual strips resident at once
constexpr int kMaxResRows = kRowsPerCta;            // residual rows of one block (all of them)
constexpr int kMaxSplit = 16;
constexpr int kMainChunkBytes = kRowsPerCta * 128;  // 8 KB
constexpr int kStripBytes = kStrip * 128;           // 2 KB
constexpr int kResChunkBytes = kResStrips * kStripBytes;
// element plane: its staged runs, per-row starts, counts and scales and the run ends live in the
// residual tile's space, which that form does not use
constexpr int kEMetaBytes = kMaxGpc * kRowsPerCta * (4 + 1 + 2) + kMaxGpc * 8;
constexpr int kEStageBytes = (kMaxChunks * kResChunkBytes - kEMetaBytes) / 16 * 16;
static_assert(kEStageBytes > 0, "element-plane staging space");
static_assert(kRowsPerCta == kElemBlock, "one element-plane block per CTA");

constexpr int kMaxGroup = kMaxGemvGroup;            // weights sharing x in one launch
constexpr int kPrefetchPerWeight = 9;
constexpr int kPrefetchRanges = kPrefetchPerWeight * kMaxGroup;

// One weight of the launch; its 64-row blocks are blockIdx.y in [block0, block0 + nb).
struct GemvWeight {
    const __half* scale1;      // [N, G]
    const __half* scale2;      // [r, G]
    const int32_t* res_slot;   // [N] or nullptr
    const __half* mu;          // [N, G] per-group offsets, or nullptr
    const uint8_t* ecount;     // element plane: [G, N] listed trits per (group, row), or nullptr
    const int32_t* ebase;      // [G * nb + 1] first listed trit of each (group, 64-row block)
    const uint8_t* eidx;       // [nnz2, padded to 16] (k % 128) << 1 | (t < 0)
    const __half* escale;      // [N, G]
    int64_t nnz2;
    __half* y;                 // [M, N]
    int64_t N, r;
    int32_t nb;                // ceil(N / 64)
    int32_t block0;
};

struct GemvMaps {
    CUtensorMap m1[kMaxGroup];     // main planes: boxes of 64 rows x 128 bytes
    CUtensorMap m2[kMaxGroup];     // residual planes: boxes of 16 rows x 128 bytes
};

struct GemvArgs {
    GemvWeight w[kMaxGroup];
    int32_t nw;
    const __half* x;           // [M, K], shared by the weights
    unsigned int* status;      // sticky timeout word
    int64_t K;
    int32_t G, M;
    int32_t gpc;               // groups per K-slice
    int32_t split;             // K-slices = cluster size
    int32_t static_weights;    // planes may be read before griddepcontrol.wait
    // byte ranges of the next call's weight to bring into L2 (16-byte aligned, sizes rounded down
    // to 16 bytes); every CTA prefetches its share of each
    // (the first npf entries; each CTA takes pf_per bytes at pf_per * its linear index)
    const uint8_t* pf_ptr[kPrefetchRanges];
    int64_t pf_bytes[kPrefetchRanges];
    int64_t pf_per[kPrefetchRanges];
    int32_t npf;
};

struct Smem {
    static constexpr int wt1 = 0;                                          // [chunk][64 rows][128 B]
    static constexpr int wt2 = wt1 + kMaxChunks * kMainChunkBytes;        // [chunk][2 strips][16][128 B]
    static constexpr int bar = wt2 + kMaxChunks * kResChunkBytes;         // mbar1[chunks], mbar2[chunks]
    static constexpr int misc = bar + (2 * kMaxChunks + 2) * 8;            // s_lo, nres (after rbar, pad)
    static constexpr int sc1 = misc + 16;                                  // half [64][kMaxGpc]
    static constexpr int sc2 = sc1 + kRowsPerCta * kMaxGpc * 2;            // half [64][kMaxGpc]
    static constexpr int bslot = sc2 + kMaxResRows * kMaxGpc * 2;          // int [64]: slot - s_lo, or -1
    static constexpr int srow = bslot + kRowsPerCta * 4;                   // int [64]: residual slot -> row
    static constexpr int cofs = srow + kMaxResRows * 4;                    // float [kMaxGpc][16]
    static constexpr int xzero = cofs + kMaxGpc * 16 * 4;                  // half [kMaxGpc * 128]: zeros
    static constexpr int smu = xzero + kMaxGpc * kGroup * 2;               // half [64][kMaxGpc]: offsets
    static constexpr int xsum = smu + kRowsPerCta * kMaxGpc * 2;           // float [kMaxGpc][16]: X_g
    static constexpr int wdesc = xsum + kMaxGpc * 16 * 4;                  // this CTA's GemvWeight
    static constexpr int red = wdesc + 128;                                // receive buffers, then xs
};
// Rows of the block owned by each rank, and the receive buffers: [rank][owned row][token] for the
// main rows' partial sums and the same for their residual rows', pushed by every rank of the cluster.
constexpr int kRecvRows = kRowsPerCta + kMaxSplit;                     // >= split * ceil(64 / split)
size_t smem_bytes(int M) {
    return size_t(Smem::red) + size_t(2 * kRecvRows) * M * 4 + size_t(M) * kMaxGpc * kGroup * 2 + 1024;
}
static_assert(Smem::xzero % 16 == 0 && Smem::red % 16 == 0, "16-byte aligned activation rows");

// One 16-row strip over the slice: yacc[t][e] += s(row) * (sum_k t * x) over the slice's groups.
// All operands are 32-bit shared addresses: box(c) is chunk c of this strip (16 rows of 128 B,
// 128-byte swizzled), sc the strip's scales [16][kMaxGpc] (fp16), xrow[t] this lane's
// activation row for token tile t (pairs in word order, or the zero row), cofs C[g][token].
// The lane holds rows rr and rr + 8. Two groups run at once, each split over two
// accumulators (the two words of the lane), so four MMA chains are in flight per warp.
// kOne: M == 1, so only the first token's elements of the accumulators are kept.
template <int NT, bool kOne, typename BoxFn, typename WaitFn>
__device__ __forceinline__ void strip_sums(int ng, int q, int rr, uint32_t sc, uint32_t cofs,
                                           const uint32_t (&xrow)[NT], BoxFn box, WaitFn wait_chunk,
                                           float (&yacc)[NT][4]) {
    // byte offset of words 2q, 2q+1 of group gl in rows rr and rr+8 (row & 7 == rr & 7):
    // chunk 2*gl + q/2 of the 128-byte row, swizzled by the row
    const int qh = q >> 1, r7 = rr & 7, qb = 8 * (q & 1);
    const uint32_t roff_a = rr * 128 + qb, roff_b = (rr + 8) * 128 + qb;
    const uint32_t sc_a = sc + rr * kMaxGpc * 2, sc_b = sc + (rr + 8) * kMaxGpc * 2;
    for (int g0 = 0; g0 < ng; g0 += 2) {
        if ((g0 % kChunkGroups) == 0) wait_chunk(g0 / kChunkGroups);
        const uint32_t b = box(g0 / kChunkGroups);          // groups g0 and g0 + 1 share a chunk
        const int ngrp = min(2, ng - g0);
        float acc[2][2][NT][4];                              // [group][word][tile][element]
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int t = 0; t < NT; ++t) acc[u][h][t][0] = acc[u][h][t][1] = acc[u][h][t][2] = acc[u][h][t][3] = 0.f;
        uint2 wa2[2], wb2[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int gl = (g0 + u) % kChunkGroups;
            const uint32_t woff = ((2 * gl + qh) ^ r7) << 4;
            wa2[u] = lds_u2(b + roff_a + woff);
            wb2[u] = lds_u2(b + roff_b + woff);
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                if (u >= ngrp) break;
                const int gi = g0 + u;
                const uint32_t wa = h ? wa2[u].y : wa2[u].x, wb = h ? wb2[u].y : wb2[u].x;
                uint32_t A[4][4];   // four MMAs per word: pairs (0,1), (2,3), (4,5), (6,7)
                decode_word_pair(wa, wb, A);
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    // the B fragments of this word's four MMAs: 32 contiguous bytes of the row
                    const uint32_t xp = xrow[t] + (gi * kGroup + 16 * (4 * h + q)) * 2;
                    const uint4 x01 = lds_u4(xp), x23 = lds_u4(xp + 16);
                    mma_16816(acc[u][h][t], A[0], x01.x, x01.y);
                    mma_16816(acc[u][h][t], A[1], x01.z, x01.w);
                    mma_16816(acc[u][h][t], A[2], x23.x, x23.y);
                    mma_16816(acc[u][h][t], A[3], x23.z, x23.w);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            if (u >= ngrp) break;
            const int gi = g0 + u;
            const float sa = lds_h2f(sc_a + gi * 2), sb = lds_h2f(sc_b + gi * 2);
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const float2 c = lds_f2(cofs + (gi * 16 + 8 * t + 2 * q) * 4);
                yacc[t][0] = fmaf(sa, (acc[u][0][t][0] + acc[u][1][t][0]) - c.x, yacc[t][0]);
                yacc[t][2] = fmaf(sb, (acc[u][0][t][2] + acc[u][1][t][2]) - c.x, yacc[t][2]);
                if (!kOne) {
                    yacc[t][1] = fmaf(sa, (acc[u][0][t][1] + acc[u][1][t][1]) - c.y, yacc[t][1]);
                    yacc[t][3] = fmaf(sb, (acc[u][0][t][3] + acc[u][1][t][3]) - c.y, yacc[t][3]);
                }
            }
        }
    }
}

// ------------------------------------------------------------------ the kernel
// kElem: the weight carries an element plane (a separate instantiation; warp 4 then sums it)
template <int NT, bool kOne, bool kElem>
__global__ void __launch_bounds__(kThreads, NT == 1 ? 6 : 3) gemv_kernel(const __grid_constant__ GemvMaps maps,
                                                                      const __grid_constant__ GemvArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    // this CTA's weight: the last whose first block is at or below blockIdx.y. Its descriptor is
    // read from a copy in shared memory (loads that may be repeated after each barrier), not
    // kept in registers for the whole kernel.
    int wi = 0;
#pragma unroll
    for (int i = 1; i < kMaxGroup; ++i)
        if (i < a.nw && int(blockIdx.y) >= a.w[i].block0) wi = i;
    static_assert(sizeof(GemvWeight) <= 120 && sizeof(GemvWeight) % 8 == 0, "descriptor slot");
    int* wsel = reinterpret_cast<int*>(smem + Smem::wdesc + 120);   // wi, for the tensor maps
    if (threadIdx.x < sizeof(GemvWeight) / 8)
        reinterpret_cast<uint64_t*>(smem + Smem::wdesc)[threadIdx.x] =
            reinterpret_cast<const uint64_t*>(&a.w[wi])[threadIdx.x];
    if (threadIdx.x == 0) *wsel = wi;
    const GemvWeight& W = *reinterpret_cast<const GemvWeight*>(smem + Smem::wdesc);
    // (the map addresses are formed where a copy is issued, from wi in shared memory)
    auto map1 = [&]() { return &maps.m1[*wsel]; };
    auto map2 = [&]() { return &maps.m2[*wsel]; };
    const int blk = int(blockIdx.y) - a.w[wi].block0;    // 64-row block within the weight
    uint8_t* wt1 = smem + Smem::wt1;
    uint8_t* wt2 = smem + Smem::wt2;
    uint64_t* mbar1 = reinterpret_cast<uint64_t*>(smem + Smem::bar);
    uint64_t* mbar2 = mbar1 + kMaxChunks;
    uint64_t* rbar = mbar2 + kMaxChunks;                 // receive barrier of the partial sums
    int* misc = reinterpret_cast<int*>(smem + Smem::misc);
    __half* sc1 = reinterpret_cast<__half*>(smem + Smem::sc1);
    __half* sc2 = reinterpret_cast<__half*>(smem + Smem::sc2);
    int* bslot = reinterpret_cast<int*>(smem + Smem::bslot);
    float* cofs = reinterpret_cast<float*>(smem + Smem::cofs);
    __half* xzero = reinterpret_cast<__half*>(smem + Smem::xzero);
    __half* smu = reinterpret_cast<__half*>(smem + Smem::smu);
    float* xsum = reinterpret_cast<float*>(smem + Smem::xsum);
    const int M = a.M;
    int* srow = reinterpret_cast<int*>(smem + Smem::srow);
    float* recv = reinterpret_cast<float*>(smem + Smem::red);                        // [split][rows/split][M]
    float* recv_res = recv + kRecvRows * M;                                          // same, residual rows
    __half* xs = reinterpret_cast<__half*>(smem + Smem::red + 2 * kRecvRows * M * 4);

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int q = lane & 3, rr = lane >> 2;
    const int ks = blockIdx.x;                        // = rank in the cluster
    const int g_begin = ks * a.gpc;
    const int ng = max(0, min(a.G, g_begin + a.gpc) - g_begin);
    const int nchunks = (ng + kChunkGroups - 1) / kChunkGroups;
    const int64_t n0 = int64_t(blk) * kRowsPerCta;
    const int xs_stride = a.gpc * kGroup;             // halves per token in smem
    bool ok = true;

    if (threadIdx.x == 0) {
        for (int c = 0; c < kMaxChunks; ++c) {
            mbar_init(&mbar1[c], 1);
            mbar_init(&mbar2[c], 1);
        }
        mbar_init(rbar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    __syncthreads();
    // this CTA has started; the matching wait comes before the first store into a peer's memory
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
    // The next call on the stream may start now: its weight loads overlap this call, and it reads
    // x (this call's output, possibly) only after griddepcontrol.wait.
    grid_launch_dependents();

    // Element plane of this block's 64 rows over the slice, staged by warp 4 with the other weight
    // reads: lane gi reads group gi's run bounds, the warp copies the runs (16-byte aligned spans)
    // into the residual tile's space with cp.async (or leaves them in global memory when they do
    // not fit), and each (group, row) cell's start, count and scale go to shared memory.
    auto elem_stage = [&]() {
        uint8_t* ebuf = wt2;
        int* estart = reinterpret_cast<int*>(wt2 + kEStageBytes);                // [kMaxGpc][64]
        uint8_t* ecnt = wt2 + kEStageBytes + kMaxGpc * kRowsPerCta * 4;          // [kMaxGpc][64]
        __half* esc = reinterpret_cast<__half*>(ecnt + kMaxGpc * kRowsPerCta);   // [kMaxGpc][64]
        int64_t* erend = reinterpret_cast<int64_t*>(esc + kMaxGpc * kRowsPerCta);  // [kMaxGpc]
        int64_t b0 = 0, b1 = 0;
        if (lane < ng) {
            const int64_t cell = int64_t(g_begin + lane) * W.nb + blk;
            b0 = min(max(int64_t(__ldg(W.ebase + cell)), int64_t(0)), W.nnz2);
            b1 = min(max(int64_t(__ldg(W.ebase + cell + 1)), b0), W.nnz2);
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int64_t n = n0 + lane + 32 * h;
            for (int gi = 0; gi < kMaxGpc; ++gi) {
                uint32_t c = 0;
                __half sc = __float2half(0.f);
                if (gi < ng && n < W.N) {
                    c = min(uint32_t(__ldg(W.ecount + int64_t(g_begin + gi) * W.N + n)), uint32_t(kGroup));
                    sc = W.escale[n * a.G + g_begin + gi];
                }
                ecnt[gi * kRowsPerCta + lane + 32 * h] = uint8_t(c);
                esc[gi * kRowsPerCta + lane + 32 * h] = sc;
            }
        }
        const int64_t a0 = b0 & ~int64_t(15), a1 = (b1 + 15) & ~int64_t(15);
        const int nchunk = lane < ng ? int((a1 - a0) >> 4) : 0;
        int coff = nchunk;                             // inclusive scan of the chunk counts
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, coff, o);
            if (lane >= o) coff += u;
        }
        const int total = __shfl_sync(0xffffffffu, coff, 31);
        coff -= nchunk;
        const bool staged = total * 16 <= kEStageBytes;
        if (staged) {
            // chunk j of the copy belongs to the last group whose first chunk is <= j
            int cof[kMaxGpc], src0[kMaxGpc];
#pragma unroll
            for (int gi = 0; gi < kMaxGpc; ++gi) {
                cof[gi] = __shfl_sync(0xffffffffu, coff, gi);
                src0[gi] = int(__shfl_sync(0xffffffffu, a0, gi) >> 4);
            }
            for (int j = lane; j < total; j += 32) {
                int from = src0[0] + j - cof[0];
#pragma unroll
                for (int q2 = 1; q2 < kMaxGpc; ++q2)
                    if (q2 < ng && cof[q2] <= j) from = src0[q2] + j - cof[q2];
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(ebuf + 16 * j)),
                             "l"(W.eidx + int64_t(from) * 16)
                             : "memory");
            }
        }
        // run base of each group in the source: the staged copy or the global list
        const int64_t rbase = staged ? int64_t(coff) * 16 + (b0 - a0) : b0;
        const int64_t rend = rbase + (b1 - b0);
        __syncwarp();
        for (int gi = 0; gi < ng; ++gi) {
            const int c0 = ecnt[gi * kRowsPerCta + lane], c1 = ecnt[gi * kRowsPerCta + 32 + lane];
            int i0 = c0, i1 = c1;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u0 = __shfl_up_sync(0xffffffffu, i0, o), u1 = __shfl_up_sync(0xffffffffu, i1, o);
                if (lane >= o) {
                    i0 += u0;
                    i1 += u1;
                }
            }
            const int tot0 = __shfl_sync(0xffffffffu, i0, 31);
            const int base = int(__shfl_sync(0xffffffffu, rbase, gi));
            const int64_t run_end = __shfl_sync(0xffffffffu, rend, gi);
            estart[gi * kRowsPerCta + lane] = base + i0 - c0;
            estart[gi * kRowsPerCta + 32 + lane] = base + tot0 + i1 - c1;
            if (lane == 0) erend[gi] = run_end;
        }
        if (lane == 0) misc[2] = staged ? 1 : 0;
    };

    int s_lo = 0, nres = 0;
    // Everything the weight determines, issued at once: TMA of the main tile (thread 0); the
    // block's residual slots, their TMA and scales (warp 4); the main scales (warps 0-3).
    auto issue_weight_reads = [&]() {
        if (threadIdx.x == 0)
            for (int c = 0; c < nchunks; ++c) {
                mbar_arrive_expect_tx(&mbar1[c], kMainChunkBytes);
                tma_load_2d(wt1 + c * kMainChunkBytes, map1(), (g_begin + c * kChunkGroups) * kWordsPerGroup,
                            int(n0), &mbar1[c]);
            }
        if (warp == kMainWarps) {
            int sl0 = -1, sl1 = -1;
            if (W.res_slot) {
                if (n0 + lane < W.N) sl0 = W.res_slot[n0 + lane];
                if (n0 + 32 + lane < W.N) sl1 = W.res_slot[n0 + 32 + lane];
            }
            const bool v0 = sl0 >= 0 && sl0 < W.r, v1 = sl1 >= 0 && sl1 < W.r;
            const unsigned b0 = __ballot_sync(0xffffffffu, v0);
            const unsigned b1 = __ballot_sync(0xffffffffu, v1);
            nres = __popc(b0) + __popc(b1);
            const int first = b0 ? (__ffs(b0) - 1) : (b1 ? 32 + __ffs(b1) - 1 : 0);
            s_lo = nres ? __shfl_sync(0xffffffffu, first < 32 ? sl0 : sl1, first & 31) : 0;
            bslot[lane] = v0 ? sl0 - s_lo : -1;
            bslot[32 + lane] = v1 ? sl1 - s_lo : -1;
            srow[lane] = -1;
            srow[32 + lane] = -1;
            __syncwarp();
            if (v0 && sl0 - s_lo < kMaxResRows) srow[sl0 - s_lo] = lane;
            if (v1 && sl1 - s_lo < kMaxResRows) srow[sl1 - s_lo] = 32 + lane;
            if (lane == 0) {
                misc[0] = s_lo;
                misc[1] = nres;
                const int strips = min(kResStrips, (nres + kStrip - 1) / kStrip);
                for (int c = 0; c < nchunks && strips > 0; ++c) {
                    mbar_arrive_expect_tx(&mbar2[c], strips * kStripBytes);
                    for (int j = 0; j < strips; ++j)
                        tma_load_2d(wt2 + c * kResChunkBytes + j * kStripBytes, map2(),
                                    (g_begin + c * kChunkGroups) * kWordsPerGroup, s_lo + j * kStrip, &mbar2[c]);
                }
            }
            if (kElem) elem_stage();
            // residual scales: lane g of each 8-lane quarter loads group g of rows quarter, +4, ...
            const int g = lane & 7;
            if (g < ng)
                for (int row = lane >> 3; row < nres; row += 4)
                    sc2[row * kMaxGpc + g] = s_lo + row < W.r ? W.scale2[int64_t(s_lo + row) * a.G + g_begin + g]
                                                              : __float2half(0.f);
        } else {
            const int g = threadIdx.x & 7;
            if (g < ng)
                for (int row = threadIdx.x >> 3; row < kRowsPerCta; row += kMainWarps * 4) {
                    const int64_t n = n0 + row;
                    sc1[row * kMaxGpc + g] = n < W.N ? W.scale1[n * a.G + g_begin + g] : __float2half(0.f);
                    if (W.mu) smu[row * kMaxGpc + g] = n < W.N ? W.mu[n * a.G + g_begin + g] : __float2half(0.f);
                }
        }
    };

    if (a.static_weights) issue_weight_reads();
    if (threadIdx.x == kThreads - 1) {
        // this CTA's share of the next call's weights, into L2
        const int64_t b = int64_t(blockIdx.y) * gridDim.x + blockIdx.x;
        for (int i = 0; i < a.npf; ++i) {
            const int64_t lo = b * a.pf_per[i], hi = min(a.pf_bytes[i], lo + a.pf_per[i]);
            if (lo < hi) prefetch_l2_bulk(a.pf_ptr[i] + lo, uint32_t(hi - lo));
        }
    }
    grid_dependency_wait();           // x (and a non-static weight) may come from the previous kernel
    if (!a.static_weights) issue_weight_reads();

    // activations of the slice, pairing columns (j, j+8) of every 16-column block; a zero row
    // stands in for the tokens past M
    {
        const int blocks16 = ng * kWordsPerGroup;
        for (int m = 0; m < M; ++m)
            for (int b = threadIdx.x; b < blocks16; b += kThreads) {
                // word b of the slice (group b / 8, word w = b % 8 = 2q + h) goes to slot 4h + q of its
                // group, so the four quad lanes of one MMA step read 128 contiguous bytes
                const int w = b & 7, slot = (b & ~7) | ((w & 1) << 2) | (w >> 1);
                const uint4* src =
                    reinterpret_cast<const uint4*>(a.x + int64_t(m) * a.K + int64_t(g_begin) * kGroup + b * 16);
                const uint4 lo = __ldg(src), hi = __ldg(src + 1);
                uint4 o0, o1;
                o0.x = prmt(lo.x, hi.x, 0x5410u); o0.y = prmt(lo.x, hi.x, 0x7632u);
                o0.z = prmt(lo.y, hi.y, 0x5410u); o0.w = prmt(lo.y, hi.y, 0x7632u);
                o1.x = prmt(lo.z, hi.z, 0x5410u); o1.y = prmt(lo.z, hi.z, 0x7632u);
                o1.z = prmt(lo.w, hi.w, 0x5410u); o1.w = prmt(lo.w, hi.w, 0x7632u);
                uint4* dst = reinterpret_cast<uint4*>(xs + size_t(m) * xs_stride + slot * 16);
                dst[0] = o0;
                dst[1] = o1;
            }
        for (int i = threadIdx.x; i < kMaxGpc * kGroup / 8; i += kThreads)
            reinterpret_cast<uint4*>(xzero)[i] = make_uint4(0u, 0u, 0u, 0u);
    }
    __syncthreads();

    uint32_t xrow[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) xrow[t] = smem_u32((8 * t + rr < M) ? xs + size_t(8 * t + rr) * xs_stride : xzero);

    // C[g][token] = sum_k (B_p(k) + 1) * x[token][k]: MMA chains on the constant pattern in the
    // same K order and with the same split into two accumulators (one per word of the lane) as
    // the main chains, combined by the same single addition, so a zero plane cancels bit for bit.
    // With one token the 8 columns of the MMA take 8 groups (column g = group g's activations),
    // so one warp computes every group's C in a single chain; each column is the same sequence
    // of operations as the per-group chains below.
    if (kOne) {
        if (warp == 0) {
            float c[2][4];
#pragma unroll
            for (int h = 0; h < 2; ++h) c[h][0] = c[h][1] = c[h][2] = c[h][3] = 0.f;
            const uint32_t xg = rr < ng ? smem_u32(xs) + rr * kGroup * 2 : smem_u32(xzero);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t xp = xg + 16 * (4 * h + q) * 2;
                const uint4 x01 = lds_u4(xp), x23 = lds_u4(xp + 16);
                uint32_t Z[4];
                zero_trit_pattern(0, Z[0], Z[2]); Z[1] = Z[0]; Z[3] = Z[2];
                mma_16816(c[h], Z, x01.x, x01.y);
                zero_trit_pattern(1, Z[0], Z[2]); Z[1] = Z[0]; Z[3] = Z[2];
                mma_16816(c[h], Z, x01.z, x01.w);
                zero_trit_pattern(2, Z[0], Z[2]); Z[1] = Z[0]; Z[3] = Z[2];
                mma_16816(c[h], Z, x23.x, x23.y);
                zero_trit_pattern(3, Z[0], Z[2]); Z[1] = Z[0]; Z[3] = Z[2];
                mma_16816(c[h], Z, x23.z, x23.w);
            }
            if (rr == 0) {   // columns 2q and 2q+1: groups 2q and 2q+1, token 0
                cofs[(2 * q) * 16] = c[0][0] + c[1][0];
                cofs[(2 * q + 1) * 16] = c[0][1] + c[1][1];
            }
        } else if (warp == 1 && W.mu) {
            // X_g = sum of the group's activations: the same chain on an all-ones A
            float c[2][4];
#pragma unroll
            for (int h = 0; h < 2; ++h) c[h][0] = c[h][1] = c[h][2] = c[h][3] = 0.f;
            const uint32_t xg = rr < ng ? smem_u32(xs) + rr * kGroup * 2 : smem_u32(xzero);
            const uint32_t one[4] = {kHalf2One, kHalf2One, kHalf2One, kHalf2One};
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t xp = xg + 16 * (4 * h + q) * 2;
                const uint4 x01 = lds_u4(xp), x23 = lds_u4(xp + 16);
                mma_16816(c[h], one, x01.x, x01.y);
                mma_16816(c[h], one, x01.z, x01.w);
                mma_16816(c[h], one, x23.x, x23.y);
                mma_16816(c[h], one, x23.z, x23.w);
            }
            if (rr == 0) {
                xsum[(2 * q) * 16] = c[0][0] + c[1][0];
                xsum[(2 * q + 1) * 16] = c[0][1] + c[1][1];
            }
        }
    } else
    for (int gi = warp; gi < ng; gi += kMainWarps + 1) {
        float c[2][NT][4];
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int t = 0; t < NT; ++t) c[h][t][0] = c[h][t][1] = c[h][t][2] = c[h][t][3] = 0.f;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const uint32_t xp = xrow[t] + (gi * kGroup + 16 * (4 * h + q)) * 2;
                const uint4 x01 = lds_u4(xp), x23 = lds_u4(xp + 16);
                uint32_t Z[4];
                zero_trit_pattern(0, Z[0], Z[2]); Z[1] = Z[0]; Z[3] = Z[2];
                mma_16816(c[h][t], Z, x01.x, x01.y);
                zero_trit_pattern(1, Z[0], Z[2]); Z[1] = Z[0]; Z[3] = Z[2];
                mma_16816(c[h][t], Z, x01.z, x01.w);
                zero_trit_pattern(2, Z[0], Z[2]); Z[1] = Z[0]; Z[3] = Z[2];
                mma_16816(c[h][t], Z, x23.x, x23.y);
                zero_trit_pattern(3, Z[0], Z[2]); Z[1] = Z[0]; Z[3] = Z[2];
                mma_16816(c[h][t], Z, x23.z, x23.w);
            }
        }
        if (rr == 0) {
#pragma unroll
            for (int t = 0; t < NT; ++t)
                *reinterpret_cast<float2*>(cofs + gi * 16 + 8 * t + 2 * q) =
                    make_float2(c[0][t][0] + c[1][t][0], c[0][t][1] + c[1][t][1]);
        }
        if (W.mu) {
            // X_g[token] = sum of the group's activations: the same chain on an all-ones A
            const uint32_t one[4] = {kHalf2One, kHalf2One, kHalf2One, kHalf2One};
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int t = 0; t < NT; ++t) c[h][t][0] = c[h][t][1] = c[h][t][2] = c[h][t][3] = 0.f;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    const uint32_t xp = xrow[t] + (gi * kGroup + 16 * (4 * h + q)) * 2;
                    const uint4 x01 = lds_u4(xp), x23 = lds_u4(xp + 16);
                    mma_16816(c[h][t], one, x01.x, x01.y);
                    mma_16816(c[h][t], one, x01.z, x01.w);
                    mma_16816(c[h][t], one, x23.x, x23.y);
                    mma_16816(c[h][t], one, x23.z, x23.w);
                }
            }
            if (rr == 0) {
#pragma unroll
                for (int t = 0; t < NT; ++t)
                    *reinterpret_cast<float2*>(xsum + gi * 16 + 8 * t + 2 * q) =
                        make_float2(c[0][t][0] + c[1][t][0], c[0][t][1] + c[1][t][1]);
            }
        }
    }
    __syncthreads();
    s_lo = misc[0];
    nres = misc[1];
    const uint32_t me = cluster_rank();
    const int rows_per_rank = (kRowsPerCta + a.split - 1) / a.split;
    const int lr0 = int(me) * rows_per_rank;
    const int nrows = max(0, min(kRowsPerCta, lr0 + rows_per_rank) - lr0);
    if (threadIdx.x == 0) {
        // every rank sends this rank M sums per owned row, and M more per owned row with a residual
        int owned_res = 0;
        for (int lo = 0; lo < nrows; ++lo) owned_res += (bslot[lr0 + lo] >= 0 && bslot[lr0 + lo] < nres) ? 1 : 0;
        if (kElem) owned_res = nrows;        // the element plane sends a sum for every row
        mbar_arrive_expect_tx(rbar, uint32_t(a.split * (nrows + owned_res) * M * 4));
    }

    // Partial sums go straight to the rank that owns the row: [this rank][row - owner's first][token]
    // in the owner's receive buffer (buf = recv for main rows, recv_res for residual rows), as
    // asynchronous stores that complete on the owner's receive barrier.
    auto push = [&](float* buf, int lrow, int t, float v) {
        const int owner = lrow / rows_per_rank;
        st_async_f32(buf + (int(me) * rows_per_rank + (lrow - owner * rows_per_rank)) * M + t, uint32_t(owner), v,
                     rbar);
    };
    // rows lrow_a and lrow_a + 8 of a strip (local rows of the block, or residual slots), this
    // lane's tokens
    auto store_red = [&](bool residual, int lrow_a, float (&yacc)[NT][4]) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            int lrow = lrow_a + 8 * h;
            if (residual) {
                if (lrow >= nres || lrow >= kMaxResRows) continue;
                lrow = srow[lrow];
                if (lrow < 0 || lrow >= kRowsPerCta) continue;   // only with an inconsistent slot map
            }
            float* buf = residual ? recv_res : recv;
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const int t0 = 8 * t + 2 * q;
                if (t0 < M) push(buf, lrow, t0, yacc[t][2 * h]);
                if (t0 + 1 < M) push(buf, lrow, t0 + 1, yacc[t][2 * h + 1]);
            }
        }
    };
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");   // every CTA of the cluster has started

    if (warp < kMainWarps) {
        float yacc[NT][4];
#pragma unroll
        for (int t = 0; t < NT; ++t) yacc[t][0] = yacc[t][1] = yacc[t][2] = yacc[t][3] = 0.f;
        const int strip_row = warp * kStrip;
        strip_sums<NT, kOne>(ng, q, rr, smem_u32(sc1 + strip_row * kMaxGpc), smem_u32(cofs), xrow,
                       [&](int c) { return smem_u32(wt1 + c * kMainChunkBytes + strip_row * 128); },
                       [&](int c) { ok = mbar_wait(&mbar1[c], 0) && ok; }, yacc);
        if (W.mu) {
            // the offset's share of the main rows: sum over the slice's groups of mu[row][g] * X_g
            const __half* ma = smu + (strip_row + rr) * kMaxGpc;
            const __half* mb = ma + 8 * kMaxGpc;
            for (int gi = 0; gi < ng; ++gi) {
                const float fa = __half2float(ma[gi]), fb = __half2float(mb[gi]);
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    const float2 xg = *reinterpret_cast<const float2*>(xsum + gi * 16 + 8 * t + 2 * q);
                    yacc[t][0] = fmaf(fa, xg.x, yacc[t][0]);
                    yacc[t][2] = fmaf(fb, xg.x, yacc[t][2]);
                    if (!kOne) {
                        yacc[t][1] = fmaf(fa, xg.y, yacc[t][1]);
                        yacc[t][3] = fmaf(fb, xg.y, yacc[t][3]);
                    }
                }
            }
        }
        store_red(false, strip_row + rr, yacc);
    } else if (nres > 0) {
        const int rounds = (nres + kResStrips * kStrip - 1) / (kResStrips * kStrip);
        for (int round = 0; round < rounds; ++round) {
            const int strips = min(kResStrips, (nres - round * kResStrips * kStrip + kStrip - 1) / kStrip);
            if (round > 0) {
                __syncwarp();                 // every lane is done with the previous round's rows
                if (lane == 0)
                    for (int c = 0; c < nchunks; ++c) {
                        mbar_arrive_expect_tx(&mbar2[c], strips * kStripBytes);
                        for (int j = 0; j < strips; ++j)
                            tma_load_2d(wt2 + c * kResChunkBytes + j * kStripBytes, map2(),
                                        (g_begin + c * kChunkGroups) * kWordsPerGroup,
                                        s_lo + (round * kResStrips + j) * kStrip, &mbar2[c]);
                    }
            }
            for (int j = 0; j < strips; ++j) {
                float yacc[NT][4];
#pragma unroll
                for (int t = 0; t < NT; ++t) yacc[t][0] = yacc[t][1] = yacc[t][2] = yacc[t][3] = 0.f;
                const int rrow = (round * kResStrips + j) * kStrip;      // first residual row of the strip
                strip_sums<NT, kOne>(ng, q, rr, smem_u32(sc2 + rrow * kMaxGpc), smem_u32(cofs), xrow,
                               [&](int c) { return smem_u32(wt2 + c * kResChunkBytes + j * kStripBytes); },
                               [&](int c) {
                                   if (j == 0) ok = mbar_wait(&mbar2[c], round & 1) && ok;
                               },
                               yacc);
                store_red(true, rrow + rr, yacc);
            }
        }
    } else if (kElem) {
        // Element plane: the runs were staged with cp.async at the start (elem_stage); M > 8: this
        // warp sums +-x over its rows' listed trits per group and scales by s2e; M <= 8: every
        // warp does, below.
        asm volatile("cp.async.wait_all;" ::: "memory");
        __syncwarp();
        if (NT == 2) {
            constexpr int kTok = 8 * NT;
            const uint8_t* src = misc[2] ? wt2 : W.eidx;
            const int* estart = reinterpret_cast<const int*>(wt2 + kEStageBytes);
            const uint8_t* ecnt = wt2 + kEStageBytes + kMaxGpc * kRowsPerCta * 4;
            const __half* esc = reinterpret_cast<const __half*>(ecnt + kMaxGpc * kRowsPerCta);
            const int64_t* erend = reinterpret_cast<const int64_t*>(esc + kMaxGpc * kRowsPerCta);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int lr = lane + 32 * h;
                float acc[kTok];
#pragma unroll
                for (int t = 0; t < kTok; ++t) acc[t] = 0.f;
                for (int gi = 0; gi < ng; ++gi) {
                    const int c = ecnt[gi * kRowsPerCta + lr], st = estart[gi * kRowsPerCta + lr];
                    const int64_t end = erend[gi];
                    float gs[kTok];
#pragma unroll
                    for (int t = 0; t < kTok; ++t) gs[t] = 0.f;
                    for (int e = 0; e < c; ++e) {
                        if (st + e >= end) break;       // only with inconsistent counts
                        const uint32_t v = src[st + e];
                        const uint32_t kk = v >> 1, w = kk >> 4, j = kk & 15;
                        const int off =
                            gi * kGroup + int((((w & 1) << 2) | (w >> 1)) * 16 + (((j & 7) << 1) | (j >> 3)));
#pragma unroll
                        for (int t = 0; t < kTok; ++t) {
                            if (t < M) {
                                const float xv = __half2float(xs[size_t(t) * xs_stride + off]);
                                gs[t] += (v & 1) ? -xv : xv;
                            }
                        }
                    }
                    const float sc = __half2float(esc[gi * kRowsPerCta + lr]);
#pragma unroll
                    for (int t = 0; t < kTok; ++t) acc[t] = fmaf(sc, gs[t], acc[t]);
                }
#pragma unroll
                for (int t = 0; t < kTok; ++t)
                    if (t < M) push(recv_res, lr, t, acc[t]);
            }
        }
    }

    if (kElem && NT == 1) {
        // Element plane, M <= 8: all 160 threads take (group, row) cells once the main strips are
        // done and warp 4's staged runs have landed; each cell's scaled sum goes to shared memory
        // (in the main tile's space, now free), then each (row, token) adds its cells in group
        // order and sends the sum to the owning rank.
        asm volatile("bar.sync 1, %0;" ::"n"(kThreads) : "memory");
        const uint8_t* ebuf = wt2;
        const int* estart = reinterpret_cast<const int*>(wt2 + kEStageBytes);
        const uint8_t* ecnt = wt2 + kEStageBytes + kMaxGpc * kRowsPerCta * 4;
        const __half* esc = reinterpret_cast<const __half*>(ecnt + kMaxGpc * kRowsPerCta);
        const int64_t* erend = reinterpret_cast<const int64_t*>(esc + kMaxGpc * kRowsPerCta);
        const uint8_t* src = misc[2] ? ebuf : W.eidx;
        float* csum = reinterpret_cast<float*>(wt1);            // [cell][M], M <= 8
        constexpr int kTok = kOne ? 1 : 8;
        for (int c = threadIdx.x; c < ng * kRowsPerCta; c += kThreads) {
            const int gi = c / kRowsPerCta;
            const int cnt = ecnt[c], st = estart[c];
            const int64_t end = erend[gi];
            float gs[kTok];
#pragma unroll
            for (int t = 0; t < kTok; ++t) gs[t] = 0.f;
            for (int e = 0; e < cnt; ++e) {
                if (st + e >= end) break;       // only with inconsistent counts
                const uint32_t v = src[st + e];
                const uint32_t kk = v >> 1, w = kk >> 4, j = kk & 15;
                const int off = gi * kGroup + int((((w & 1) << 2) | (w >> 1)) * 16 + (((j & 7) << 1) | (j >> 3)));
#pragma unroll
                for (int t = 0; t < kTok; ++t) {
                    if (t < M) {
                        const float xv = __half2float(xs[size_t(t) * xs_stride + off]);
                        gs[t] += (v & 1) ? -xv : xv;
                    }
                }
            }
            const float sc = __half2float(esc[c]);
#pragma unroll
            for (int t = 0; t < kTok; ++t)
                if (t < M) csum[c * M + t] = sc * gs[t];
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kThreads) : "memory");
        for (int i = threadIdx.x; i < kRowsPerCta * M; i += kThreads) {
            const int lr = i % kRowsPerCta, t = i / kRowsPerCta;
            float sum = 0.f;
            for (int gi = 0; gi < ng; ++gi) sum += csum[(gi * kRowsPerCta + lr) * M + t];
            push(recv_res, lr, t, sum);
        }
    }

    // Epilogue: once the partial sums of this rank's rows have arrived from every rank (the
    // receive barrier counts their bytes) they are summed in rank order, the residual rows' sums
    // added, and rounded once. No CTA reads another's memory, so none waits for its peers to end.
    // The wait runs whatever `ok` is: every rank pushes its partial sums on every path, and a CTA
    // that left early would take stores into the shared memory of an exited CTA.
    ok = mbar_wait(rbar, 0) && ok;
    {
        for (int i = threadIdx.x; i < nrows * M; i += kThreads) {
            const int tok = i / nrows, lo = i - tok * nrows, lr = lr0 + lo;
            const int64_t n = n0 + lr;
            if (n >= W.N) continue;
            float s = 0.f;
            for (int c = 0; c < a.split; ++c) s += recv[(c * rows_per_rank + lo) * M + tok];
            const int slot = bslot[lr];
            if (kElem || (slot >= 0 && slot < nres)) {
                float s2 = 0.f;
                for (int c = 0; c < a.split; ++c) s2 += recv_res[(c * rows_per_rank + lo) * M + tok];
                s += s2;
            }
            W.y[int64_t(tok) * W.N + n] = __float2half_rn(s);
        }
    }
    if (!ok && a.status) atomicOr(a.status, 1u);
}

// ------------------------------------------------------------------ host side
int env_split() {
    static int v = [] {
        const char* s = getenv("TERN_SPLITK");
        return s ? atoi(s) : 0;
    }();
    return v;
}

struct Plan {
    int split, gpc;
};

Plan plan_for(int64_t blocks, int64_t K) {
    const int G = int(K / kGroup);
    const int min_split = (G + kMaxGpc - 1) / kMaxGpc;
    const int64_t target = 4LL * sm_count();
    const int par = int(std::min<int64_t>(kMaxSplit, (target + blocks - 1) / blocks));
    int split = std::max(min_split, env_split() > 0 ? env_split() : par);
    split = std::max(1, std::min(split, std::min(kMaxSplit, G)));
    Plan p;
    p.gpc = (G + split - 1) / split;
    p.split = (G + p.gpc - 1) / p.gpc;
    return p;
}

template <int NT, bool kOne, bool kElem>
tern_status launch(const GemvMaps& maps, const GemvArgs& args, int64_t blocks, size_t smem, cudaStream_t stream) {
    auto kernel = gemv_kernel<NT, kOne, kElem>;
    static std::mutex mu;
    static bool configured[64] = {false};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return TERN_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!configured[dev]) {
            if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 160 * 1024) != cudaSuccess ||
                cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
                return TERN_ERR_CUDA;
            configured[dev] = true;
        }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(args.split), unsigned(blocks), 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = unsigned(args.split);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, kernel, maps, args) != cudaSuccess) return TERN_ERR_CUDA;
    return TERN_OK;
}

}  // namespace

size_t gemv_workspace_bytes(const tern_weight&, int64_t) { return 0; }

tern_status gemv_launch_group(const tern_weight* const* ws, int nw, const __half* x, int M, __half* const* ys,
                              const tern_weight* const* next, int nnext, cudaStream_t stream) {
    if (nw < 1 || nw > kMaxGroup || nnext < 0 || nnext > kMaxGroup) return TERN_ERR_SHAPE;
    GemvMaps maps;
    GemvArgs a = {};
    int64_t blocks = 0;
    bool elem = false, all_static = true;
    for (int i = 0; i < nw; ++i) {
        const tern_weight& w = *ws[i];
        if (w.K != ws[0]->K) return TERN_ERR_SHAPE;
        if (!plane_map(&maps.m1[i], w.plane1, w.N, w.K, 32, kRowsPerCta, CU_TENSOR_MAP_SWIZZLE_128B))
            return TERN_ERR_CUDA;
        if (!plane_map(&maps.m2[i], w.r > 0 ? w.plane2 : w.plane1, w.r > 0 ? w.r : w.N, w.K, 32, kStrip,
                       CU_TENSOR_MAP_SWIZZLE_128B))
            return TERN_ERR_CUDA;
        GemvWeight& g = a.w[i];
        g.scale1 = reinterpret_cast<const __half*>(w.scale1);
        g.scale2 = reinterpret_cast<const __half*>(w.scale2);
        g.res_slot = w.r > 0 ? w.res_slot : nullptr;
        g.mu = reinterpret_cast<const __half*>(w.mu);
        if (w.ecount) {
            g.ecount = w.ecount;
            g.ebase = w.ebase;
            g.eidx = w.eidx;
            g.escale = reinterpret_cast<const __half*>(w.escale);
            g.nnz2 = w.nnz2;
            elem = true;
        }
        g.y = ys[i];
        g.N = w.N;
        g.r = w.r;
        g.nb = int32_t((w.N + kRowsPerCta - 1) / kRowsPerCta);
        g.block0 = int32_t(blocks);
        blocks += g.nb;
        all_static = all_static && (w.flags & TERN_WEIGHT_STATIC);
    }
    if (blocks > 65535) return TERN_ERR_SHAPE;
    const Plan p = plan_for(blocks, ws[0]->K);
    a.nw = nw;
    a.x = x;
    a.status = async_status_word();
    a.K = ws[0]->K;
    a.G = int32_t(ws[0]->K / kGroup);
    a.M = M;
    a.gpc = p.gpc;
    a.split = p.split;
    a.static_weights = all_static ? 1 : 0;
    for (int j = 0; j < nnext; ++j) {
        const tern_weight* nx = next[j];
        const int64_t G = nx->K / kGroup, rn = nx->r;
        const bool ne = nx->ecount != nullptr;
        const void* ptr[kPrefetchPerWeight] = {nx->plane1, nx->scale1, rn > 0 ? nx->res_slot : nullptr,
                                               rn > 0 ? nx->plane2 : nullptr, rn > 0 ? nx->scale2 : nullptr,
                                               nx->mu, ne ? nx->ecount : nullptr, ne ? nx->eidx : nullptr,
                                               ne ? nx->escale : nullptr};
        const int64_t bytes[kPrefetchPerWeight] = {nx->N * (nx->K / 4), nx->N * G * 2, nx->N * 4, rn * (nx->K / 4),
                                                   rn * G * 2, nx->N * G * 2, nx->N * G, ne ? nx->nnz2 : 0,
                                                   nx->N * G * 2};
        for (int i = 0; i < kPrefetchPerWeight; ++i) {
            const int64_t b16 = bytes[i] / 16 * 16;
            if (!ptr[i] || b16 <= 0) continue;
            a.pf_ptr[a.npf] = static_cast<const uint8_t*>(ptr[i]);
            a.pf_bytes[a.npf] = b16;
            ++a.npf;
        }
    }
    const int64_t nctas = int64_t(p.split) * blocks;
    for (int i = 0; i < a.npf; ++i) a.pf_per[i] = ((a.pf_bytes[i] + nctas - 1) / nctas + 15) / 16 * 16;
    const size_t smem = smem_bytes(M);
    if (elem) {
        if (M == 1) return launch<1, true, true>(maps, a, blocks, smem, stream);
        return M <= 8 ? launch<1, false, true>(maps, a, blocks, smem, stream)
                      : launch<2, false, true>(maps, a, blocks, smem, stream);
    }
    if (M == 1) return launch<1, true, false>(maps, a, blocks, smem, stream);
    return M <= 8 ? launch<1, false, false>(maps, a, blocks, smem, stream)
                  : launch<2, false, false>(maps, a, blocks, smem, stream);
}

}  // namespace tern
