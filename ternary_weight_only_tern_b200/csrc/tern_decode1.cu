// Decode GEMV for one token (M = 1): y[N] = x[K] . W^T with W on packed 2-bit ternary planes.
//
// What it computes is the representation of "Post-Training Ternarization of Qwen3-4B"
// (arXiv 2609.01962v1), sections 4.3-4.5: one ternary plane T1 with an fp16 scale per
// (row, 128-wide K group), a residual plane T2 with its own scales on a sorted subset R of rows,
// optionally a per-group offset mu (section 4.3's asymmetric offset); activations stay fp16
// (section 3.1). With t in {-1, 0, +1} every product t*x is exact, so the layer is a signed sum
// of activations ("Can Ternary LLMs Hit 1.58 Bits per Weight?", promptzone, "What It Is and How
// It Works"), accumulated here in fp32 and rounded to fp16 once.
//
// Design (B200; a stream of 0.27 bytes per weight that must run at HBM speed):
//  * Persistent grid, one CTA per SM. The 16-row strips of all weights of the launch are split
//    into contiguous ranges that differ by at most one strip, one per CTA, so every output row is
//    finished inside one CTA: no partial sum leaves the SM and no workspace is needed.
//  * Warp-specialised CTA. A bulk or TMA copy holds its issuing thread until the copy before it
//    has landed, so four producer warps issue the strips' planes (one 3D TMA box each: 16 rows x
//    up to SB 512-wide K slabs, 128-byte swizzle, no multicast) and four more the strips' scales
//    and offsets (one bulk copy each), every one taking every fourth stage of a ring of NS. W
//    consumer warps each own a fixed share of the K groups of every stage; once a warp has its
//    words and scales in registers the stage is free again. An epilogue warp adds the consumers'
//    partial sums in warp order, keeps the sums of the current segment (up to 256 rows) in shared
//    memory, adds the residual rows' sums and writes y.
//  * Residual rows: since R is sorted, the residual rows of a segment are the contiguous slots
//    [s_a, s_a + span) of the residual plane; they stream as extra 16-slot strips after the
//    segment's main strips, and each row's residual sum joins its main sum before the single
//    rounding to fp16.
//  * The signed sums run on the tensor pipe as mma.sync m16n8k16 (fp16 in, fp32 accumulate),
//    A = 16 weight rows x 16 K of decoded trits. With one token, each of a warp's (up to 4)
//    groups keeps the token in its own MMA column: lanes of row index rr = 2 g hold group g's
//    activations, so one set of 16 activation registers per lane serves all of the warp's
//    groups, and each group accumulates in its own registers, whose column 2 g alone is read
//    (the other columns multiply other groups' activations and are ignored). Lane q then holds
//    group q's sums for its two rows, and the per-group scaling costs a few instructions per
//    32 MMAs. The groups' MMA chains are interleaved step by step with their decode.
//  * Decode is branch-free: one LOP3 writes two 2-bit codes (trits p and p+8 of a word) into
//    the mantissas of an fp16 pair (B_p + c); pairs 0-4 read the codes in place and pairs 5-7
//    after one shift of the word (tern_device.cuh); the MMA sums (B_p + 1 + t) x,
//    and C = sum (B_p + 1) x, computed once per kernel by the same MMA chain on the constant
//    pattern, is subtracted once per group, so a zero plane cancels bit for bit. With an offset,
//    the group sums X_g come from the same chain on an all-ones pattern.
//  * x is staged once per CTA in shared memory with the two activations of each decoded pair
//    adjacent (pair p of word w = activations 16 w + p and 16 w + p + 8).
//  * Programmatic dependent launch: the CTA lets the next kernel launch at once; with static
//    weights its weight and slot-map reads start before griddepcontrol.wait, x is read and y is
//    written only after it.
//  * Every wait is bounded; a wait that runs out records TERN_ERR_TIMEOUT in the sticky status
//    word and the warps leave their loops; the producers first wait, again bounded, for the TMA
//    copies they issued.
#include <algorithm>
#include <mutex>

#include "tern_device.cuh"

namespace tern {
namespace {

using namespace dev;

constexpr int kStrip = 16;                 // rows per strip (the MMA's M)
constexpr int kSegStrips = 16;             // strips per segment
constexpr int kSegRows = kSegStrips * kStrip;
constexpr int kMaxSegs = 8;                // segments per CTA
constexpr int kSlabTile = kStrip * 128;    // bytes of one strip's slab: 16 rows x 128 B
constexpr int kMaxNW = kMaxGemvGroup;      // weights per launch
// A bulk or TMA copy holds its issuing thread until the copy before it has landed, so the bytes
// in flight are (issuing threads) x (bytes per copy). Four warps issue the planes' boxes and four
// the scales' (and offsets') runs, each taking every fourth stage.
constexpr int kIssuePerKind = 4;
constexpr int kStages = 8;                 // ring stages (fewer when shared memory runs short)
constexpr int kProducers = 2 * kIssuePerKind;
constexpr int kPfPerWeight = 6;
constexpr int kPfRanges = kPfPerWeight * kMaxNW;

struct D1Weight {
    const __half* scale1;     // [N, G]
    const __half* scale2;     // [r, G]
    const int32_t* res_slot;  // [N] or nullptr (r == 0)
    const __half* mu;         // [N, G] or nullptr
    __half* y;                // [N]
    int64_t N, r;
    int32_t strip0, nstrips;  // this weight's strips are [strip0, strip0 + nstrips) of the launch
};

struct D1Maps {
    CUtensorMap m1[kMaxNW];   // plane1 viewed as [slab][row][32 words]: box {32, 16, SB}
    CUtensorMap m2[kMaxNW];   // plane2, the same
};

struct D1Args {
    D1Weight w[kMaxNW];
    int32_t nw;
    const __half* x;          // [K]
    unsigned int* status;
    int32_t K, G;
    int32_t SB;               // slabs per stage (per TMA box)
    int32_t nchunk;           // stages per strip = ceil(K / (512 SB))
    int32_t NS;               // ring stages
    int32_t S;                // strips of the launch
    int32_t static_weights;
    int32_t has_mu;
    // shared-memory offsets in bytes from the 1024-aligned base (the stages start at 0)
    int32_t o_sc, o_mu, o_red, o_xs, o_cofs, o_xsum, o_meta, o_bslot, o_mainy, o_resy, o_bar;
    // L2 prefetch of the next call's weights: each CTA takes pf_per bytes of each range
    const uint8_t* pf_ptr[kPfRanges];
    int64_t pf_bytes[kPfRanges];
    int64_t pf_per[kPfRanges];
    int32_t npf;
};

struct Seg {
    int wi;        // weight
    int ja, jb;    // strips [ja, jb) of the weight
};

// The next segment of the strip range [j, j1): at most kSegStrips strips of one weight.
__device__ __forceinline__ bool next_seg(const D1Args& a, int& j, int j1, Seg& s) {
    if (j >= j1) return false;
    int wi = 0;
#pragma unroll
    for (int i = 1; i < kMaxNW; ++i)
        if (i < a.nw && j >= a.w[i].strip0) wi = i;
    const int base = a.w[wi].strip0;
    const int jb = min(min(j1, base + a.w[wi].nstrips), j + kSegStrips);
    s.wi = wi;
    s.ja = j - base;
    s.jb = jb - base;
    j = jb;
    return true;
}

// Every role walks the same job sequence: per segment, its main strips (nchunk stages each),
// then its residual strips (known once the epilogue warp has published the segment metadata).
// fn(kind, segment index, segment, strip within the kind, chunk) returns false to stop.
template <typename Fn, typename MetaWait>
__device__ __forceinline__ void walk_jobs(const D1Args& a, int j0, int j1, const int* meta, MetaWait meta_wait,
                                          Fn fn) {
    int j = j0, k = 0;
    Seg sg;
    bool have_meta = false;
    while (k < kMaxSegs && next_seg(a, j, j1, sg)) {
        for (int jj = sg.ja; jj < sg.jb; ++jj)
            for (int c = 0; c < a.nchunk; ++c)
                if (!fn(0, k, sg, jj, c)) return;
        if (!have_meta) {
            if (!meta_wait()) return;
            have_meta = true;
        }
        const int nrs = meta[2 * k + 1];
        for (int t = 0; t < nrs; ++t)
            for (int c = 0; c < a.nchunk; ++c)
                if (!fn(1, k, sg, t, c)) return;
        ++k;
    }
}

// 1D bulk copy global -> this CTA's shared memory (16-byte aligned, bytes a multiple of 16),
// completing as transaction bytes on `bar`.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// The scales of rows [row0, row0 + rows) of a [*, G] fp16 array are one contiguous run. They
// reach shared memory at dst as one bulk copy from the 16-byte boundary at or below the run's start
// (the run then begins `skew` bytes into dst) and, for the last bytes that do not fill 16, plain
// loads and stores. stage_plan writes those last bytes and returns the bulk copy's source offset
// and size; stage_issue issues it (after the barrier expects its bytes).
struct RowRun {
    uint64_t a0;      // byte offset of the bulk copy's source
    uint32_t bytes;   // bulk copy size (a multiple of 16, may be 0)
};

__device__ __forceinline__ RowRun stage_plan(uint32_t dst, const __half* base, int64_t row0, int rows, int G) {
    RowRun r{0, 0};
    if (rows <= 0) return r;
    const uint64_t start = uint64_t(row0) * G * 2, end = start + uint64_t(rows) * G * 2;
    const uint64_t a0 = start & ~uint64_t(15), a1 = end & ~uint64_t(15);
    const uint8_t* src = reinterpret_cast<const uint8_t*>(base);
    for (uint64_t b = a1; b < end; b += 2) {
        const unsigned short h = __ldg(reinterpret_cast<const unsigned short*>(src + b));
        asm volatile("st.shared.u16 [%0], %1;" ::"r"(dst + uint32_t(b - a0)), "h"(h) : "memory");
    }
    r.a0 = a0;
    r.bytes = uint32_t(a1 - a0);
    return r;
}

__device__ __forceinline__ void stage_issue(uint32_t dst, const __half* base, RowRun r, uint64_t* bar) {
    if (r.bytes) bulk_load(dst, reinterpret_cast<const uint8_t*>(base) + r.a0, r.bytes, bar);
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 3D tiled TMA load (no multicast) into this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int c0, int c1, int c2,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
        : "memory");
}

// Bounded wait that polls the barrier with the non-blocking test_wait: a warp suspended in
// try_wait was measured to resume about a microsecond after the phase completed, which at this
// kernel's stage rate costs more than the issue slots the polling takes.
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t* bar, uint32_t parity) {
    const uint32_t addr = smem_u32(bar);
    uint64_t t0 = 0;
    for (uint32_t i = 0;; ++i) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(addr), "r"(parity)
            : "memory");
        if (done) return true;
        const uint64_t t = clock64();
        if (i == 0) t0 = t;
        else if (t - t0 > kWaitLimitCycles) return false;
    }
}

__device__ __forceinline__ float sel4(int q, float a0, float a1, float a2, float a3) {
    const float lo = (q & 1) ? a1 : a0, hi = (q & 1) ? a3 : a2;
    return (q & 2) ? hi : lo;
}

// Groups [g0, g0 + ng) of a chunk of gc groups belong to consumer warp w of W.
__device__ __forceinline__ void warp_groups(int gc, int w, int W, int& g0, int& ng) {
    g0 = (w * gc) / W;
    ng = ((w + 1) * gc) / W - g0;
}

// Lane rows: lane row index rr of the MMA handles strip rows pi(rr) and pi(rr) + 8, with
// pi = 0, 2, 4, 6, 1, 3, 5, 7, so that each half-warp's 8-byte reads of the 128-byte-swizzled
// tile fall in 32 distinct banks.
__device__ __forceinline__ int lane_row(int rr) { return rr < 4 ? 2 * rr : 2 * (rr - 4) + 1; }

// W consumer warps; GW groups per warp per stage (a warp with fewer groups in a stage repeats
// its last one and discards the extra sums).
template <int W, int GW>
__global__ void __launch_bounds__((W + kProducers + 1) * 32, 1) decode1_kernel(const __grid_constant__ D1Maps maps,
                                                                  const __grid_constant__ D1Args a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int NS = a.NS, SB = a.SB, nchunk = a.nchunk;
    const int gcmax = 4 * SB;                                   // groups per full chunk
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + a.o_bar);
    uint64_t* redfull = full + NS;
    uint64_t* empty = redfull + NS;                             // the stage's tile and scales are free
    uint64_t* redempty = empty + NS;                            // the stage's partial sums were read
    uint64_t* meta_bar = redempty + NS;
    int* abort_flag = reinterpret_cast<int*>(meta_bar + 1);
    const uint32_t stage0 = smem_u32(smem);
    const int stage_bytes = SB * kSlabTile;
    const int sc_stride = (32 * a.G + 16 + 15) & ~15;          // bytes per stage: 16 rows x G, + skew
    uint8_t* sc_base = smem + a.o_sc;                            // [NS][16 rows][G] fp16 (skewed)
    uint8_t* mu_base = smem + a.o_mu;                            // [NS][16 rows][G] fp16
    float* red = reinterpret_cast<float*>(smem + a.o_red);       // [NS][W][4 groups][16 rows]
    __half* xs = reinterpret_cast<__half*>(smem + a.o_xs);       // [K], pairs adjacent
    float* cofs = reinterpret_cast<float*>(smem + a.o_cofs);     // [nchunk][W][4]
    float* xsum = reinterpret_cast<float*>(smem + a.o_xsum);     // [nchunk][W][4]
    int* meta = reinterpret_cast<int*>(smem + a.o_meta);         // [kMaxSegs][2]: s_a, residual strips
    int16_t* bslot = reinterpret_cast<int16_t*>(smem + a.o_bslot);  // [kMaxSegs][256]
    float* main_y = reinterpret_cast<float*>(smem + a.o_mainy);  // [256]
    float* res_y = reinterpret_cast<float*>(smem + a.o_resy);    // [256]

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 2);             // the plane's issuer and the scales' issuer
            mbar_init(&redfull[s], W);
            mbar_init(&empty[s], W);
            mbar_init(&redempty[s], 1);
        }
        mbar_init(meta_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    grid_launch_dependents();

    const int P = gridDim.x, b = blockIdx.x;
    const int j0 = int((int64_t(b) * a.S) / P), j1 = int((int64_t(b + 1) * a.S) / P);
    volatile int* vabort = abort_flag;
    auto fail = [&]() {
        *vabort = 1;
        if (a.status) atomicOr(a.status, 1u);
    };
    auto meta_wait = [&]() -> bool {
        if (mbar_wait_sleep(meta_bar, 0)) return true;
        fail();
        return false;
    };

    if (warp >= W && warp < W + kProducers) {
        // ------------------------------------------------------------ producers
        // producer warp p < kIssuePerKind issues the planes of the jobs u with
        // u % kIssuePerKind == p, warp kIssuePerKind + p their scales and offsets
        const int pw = (warp - W) % kIssuePerKind;
        const bool planes = (warp - W) < kIssuePerKind;
        if (warp == W && lane < a.nw) {
            prefetch_tensormap(&maps.m1[lane]);
            prefetch_tensormap(&maps.m2[lane]);
        }
        if (!a.static_weights) grid_dependency_wait();
        int job = 0, last_mine = -1;
        walk_jobs(a, j0, j1, meta, meta_wait, [&](int kind, int k, const Seg& sg, int jj, int c) -> bool {
            if (*vabort) return false;
            if (job % kIssuePerKind != pw) {
                ++job;
                return true;
            }
            last_mine = job;
            const D1Weight& Wt = a.w[sg.wi];
            const int s = job % NS, round = job / NS;
            if (round > 0 && !mbar_wait_sleep(&empty[s], (round - 1) & 1)) {
                fail();
                return false;
            }
            const CUtensorMap* map = kind ? &maps.m2[sg.wi] : &maps.m1[sg.wi];
            const int64_t row0 = kind ? int64_t(meta[2 * k]) + int64_t(jj) * kStrip : int64_t(jj) * kStrip;
            const int64_t nrows = kind ? Wt.r : Wt.N;
            const __half* scale = kind ? Wt.scale2 : Wt.scale1;
            const __half* mu = kind == 0 ? Wt.mu : nullptr;
            if (lane == 0 && planes) {
                // the strip's plane: one TMA box, counted as transaction bytes on the barrier
                mbar_arrive_expect_tx(&full[s], uint32_t(stage_bytes));
                tma_load_3d(stage0 + s * stage_bytes, map, 0, int(row0), c * SB, &full[s]);
            } else if (lane == 0) {
                // its 16 rows of scales (and offsets); the barrier expects the bytes first
                const int rows = int(max(int64_t(0), min(int64_t(kStrip), nrows - row0)));
                const uint32_t scd = smem_u32(sc_base + s * sc_stride), mud = smem_u32(mu_base + s * sc_stride);
                const RowRun rs = stage_plan(scd, scale, row0, rows, a.G);
                const RowRun rm = mu ? stage_plan(mud, mu, row0, rows, a.G) : RowRun{0, 0};
                mbar_arrive_expect_tx(&full[s], rs.bytes + rm.bytes);
                stage_issue(scd, scale, rs, &full[s]);
                if (mu) stage_issue(mud, mu, rm, &full[s]);
            }
            ++job;
            return true;
        });
        // the next call's weights into L2 (a hint), then wait for the copies still in flight
        if (lane == 0 && warp == W) {
            for (int i = 0; i < a.npf; ++i) {
                const int64_t lo = int64_t(b) * a.pf_per[i], hi = min(a.pf_bytes[i], lo + a.pf_per[i]);
                if (lo < hi) prefetch_l2_bulk(a.pf_ptr[i] + lo, uint32_t(hi - lo));
            }
        }
        for (int u = max(0, job - NS); u <= last_mine; ++u)
            if (u % kIssuePerKind == pw && !mbar_wait(&full[u % NS], (u / NS) & 1)) break;
        return;
    }

    if (warp == W + kProducers) {
        // ------------------------------------------------------------ epilogue
        // segment metadata: the slots of the segment's residual rows
        if (!a.static_weights) grid_dependency_wait();
        {
            int j = j0, k = 0;
            Seg sg;
            while (k < kMaxSegs && next_seg(a, j, j1, sg)) {
                const D1Weight& Wt = a.w[sg.wi];
                const int64_t n_a = int64_t(sg.ja) * kStrip;
                const int rows = int(min(int64_t(sg.jb) * kStrip, Wt.N) - n_a);
                int smin = 0x7fffffff, smax = -1;
                int sl[kSegRows / 32];
#pragma unroll
                for (int i = 0; i < kSegRows / 32; ++i) {
                    const int lr = lane + 32 * i;
                    int v = -1;
                    if (Wt.res_slot && Wt.r > 0 && lr < rows) v = __ldg(Wt.res_slot + n_a + lr);
                    if (v >= Wt.r) v = -1;
                    sl[i] = v;
                    if (v >= 0) {
                        smin = min(smin, v);
                        smax = max(smax, v);
                    }
                }
                smin = __reduce_min_sync(0xffffffffu, smin);
                smax = __reduce_max_sync(0xffffffffu, smax);
                const int span = smax >= 0 ? min(smax - smin + 1, kSegRows) : 0;
#pragma unroll
                for (int i = 0; i < kSegRows / 32; ++i) {
                    const int d = sl[i] - smin;
                    bslot[k * kSegRows + lane + 32 * i] = int16_t((sl[i] >= 0 && d < span) ? d : -1);
                }
                if (lane == 0) {
                    meta[2 * k] = smax >= 0 ? smin : 0;
                    meta[2 * k + 1] = (span + kStrip - 1) / kStrip;
                }
                ++k;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(meta_bar);
        }
        grid_dependency_wait();       // y may still be read by the previous kernel
        int job = 0;
        int cur_k = -1;
        Seg cur{};
        auto flush = [&]() {          // write the finished segment's rows
            if (cur_k < 0) return;
            const D1Weight& Wt = a.w[cur.wi];
            const int64_t n_a = int64_t(cur.ja) * kStrip;
            const int rows = int(min(int64_t(cur.jb) * kStrip, Wt.N) - n_a);
            __syncwarp();
            for (int lr = lane; lr < rows; lr += 32) {
                float v = main_y[lr];
                const int bs = bslot[cur_k * kSegRows + lr];
                if (bs >= 0) v += res_y[bs];
                Wt.y[n_a + lr] = __float2half_rn(v);
            }
            __syncwarp();
        };
        walk_jobs(a, j0, j1, meta, [] { return true; }, [&](int kind, int k, const Seg& sg, int jj, int c) -> bool {
            if (*vabort) return false;
            if (k != cur_k) {
                flush();
                cur_k = k;
                cur = sg;
            }
            const int s = job % NS, round = job / NS;
            if (!mbar_wait_sleep(&redfull[s], round & 1)) {
                fail();
                return false;
            }
            if (lane < kStrip) {
                float v = 0.f;
                // every consumer warp's group sums, in warp order, then group order
                for (int w = 0; w < W; ++w)
#pragma unroll
                    for (int g = 0; g < 4; ++g) v += red[((s * W + w) * 4 + g) * kStrip + lane];
                const int idx = kind ? jj * kStrip + lane : (jj - sg.ja) * kStrip + lane;
                float* dst = kind ? res_y : main_y;
                dst[idx] = c ? dst[idx] + v : v;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&redempty[s]);
            ++job;
            return true;
        });
        if (!*vabort) flush();
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int q = lane & 3, rr = lane >> 2;
    const int pr = lane_row(rr);
    grid_dependency_wait();
    // stage x with the two activations of each pair adjacent
    for (int i = threadIdx.x; i < a.K / 16; i += W * 32) {
        const uint4* src = reinterpret_cast<const uint4*>(a.x + int64_t(i) * 16);
        const uint4 lo = __ldg(src), hi = __ldg(src + 1);
        uint4 o0, o1;
        o0.x = prmt(lo.x, hi.x, 0x5410u); o0.y = prmt(lo.x, hi.x, 0x7632u);
        o0.z = prmt(lo.y, hi.y, 0x5410u); o0.w = prmt(lo.y, hi.y, 0x7632u);
        o1.x = prmt(lo.z, hi.z, 0x5410u); o1.y = prmt(lo.z, hi.z, 0x7632u);
        o1.z = prmt(lo.w, hi.w, 0x5410u); o1.w = prmt(lo.w, hi.w, 0x7632u);
        uint4* dst = reinterpret_cast<uint4*>(xs + int64_t(i) * 16);
        dst[0] = o0;
        dst[1] = o1;
    }
    asm volatile("bar.sync 1, %0;" ::"n"(W * 32) : "memory");

    // The lane's activation registers for chunk c: words 2q, 2q+1 of the warp's group rr / 2
    // (group 0 of the warp for the lanes whose column is not read).
    uint32_t xr[16];
    auto load_x = [&](int c) {
        int g0, ng;
        warp_groups(min(gcmax, a.G - c * gcmax), warp, W, g0, ng);
        const int gl = (rr & 1) == 0 && (rr >> 1) < ng ? (rr >> 1) : 0;
        const uint32_t src = smem_u32(xs) + uint32_t(((c * gcmax + g0 + gl) * kGroup + 32 * q) * 2);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 v = lds_u4(src + 16 * i);
            xr[4 * i] = v.x; xr[4 * i + 1] = v.y; xr[4 * i + 2] = v.z; xr[4 * i + 3] = v.w;
        }
    };
    // C and X of every chunk's groups of this warp: one MMA chain each on the constant patterns
    for (int c = 0; c < nchunk; ++c) {
        load_x(c);
        // the same chain as the main sums (both words of the lane into one accumulator)
        float cz[4] = {}, co[4] = {};
        const uint32_t one[4] = {kHalf2One, kHalf2One, kHalf2One, kHalf2One};
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint32_t Z[4];
                zero_trit_pattern_in_place(i, Z[0], Z[2]);
                Z[1] = Z[0];
                Z[3] = Z[2];
                mma_16816(cz, Z, xr[8 * h + 2 * i], xr[8 * h + 2 * i + 1]);
                if (a.has_mu) mma_16816(co, one, xr[8 * h + 2 * i], xr[8 * h + 2 * i + 1]);
            }
        if (rr == 0) {     // column 2q: group q of the warp
            cofs[(c * W + warp) * 4 + q] = cz[0];
            xsum[(c * W + warp) * 4 + q] = co[0];
        }
    }
    __syncwarp();
    if (nchunk == 1) load_x(0);
    if (!meta_wait()) return;

    struct Sc {
        unsigned short sa, sb, ma, mb;
    };
    // A job's accumulators and what its epilogue (per-group scaling and the hand-off of each
    // lane's two row sums of its group to the epilogue warp, which adds them) needs.
    struct Pending {
        float acc[4][4];
        Sc sc;
        int s, round, c, ng, mu;
    };
    auto finish = [&](const Pending& pd) -> bool {
        float p0 = 0.f, p1 = 0.f;
        if (q < pd.ng) {
            const float v0 = sel4(q, pd.acc[0][0], pd.acc[1][0], pd.acc[2][0], pd.acc[3][0]);
            const float v1 = sel4(q, pd.acc[0][2], pd.acc[1][2], pd.acc[2][2], pd.acc[3][2]);
            const float C = cofs[(pd.c * W + warp) * 4 + q];
            p0 = __half2float(__ushort_as_half(pd.sc.sa)) * (v0 - C);
            p1 = __half2float(__ushort_as_half(pd.sc.sb)) * (v1 - C);
            if (pd.mu) {
                const float X = xsum[(pd.c * W + warp) * 4 + q];
                p0 = fmaf(__half2float(__ushort_as_half(pd.sc.ma)), X, p0);
                p1 = fmaf(__half2float(__ushort_as_half(pd.sc.mb)), X, p1);
            }
        }
        if (pd.round > 0 && !mbar_wait_sleep(&redempty[pd.s], (pd.round - 1) & 1)) {
            fail();
            return false;
        }
        float* rq = red + ((pd.s * W + warp) * 4 + q) * kStrip;
        rq[pr] = p0;
        rq[pr + 8] = p1;
        __syncwarp();
        if (lane == 0) mbar_arrive(&redfull[pd.s]);
        return true;
    };

    int job = 0;
    walk_jobs(a, j0, j1, meta, meta_wait, [&](int kind, int k, const Seg& sg, int jj, int c) -> bool {
        if (*vabort) return false;
        const int s = job % NS, round = job / NS;
        int g0, ng;
        const int gc = min(gcmax, a.G - c * gcmax);
        warp_groups(gc, warp, W, g0, ng);
        if (nchunk > 1) load_x(c);
        if (!mbar_wait_sleep(&full[s], round & 1)) {
            fail();
            return false;
        }
        const uint32_t tile = stage0 + s * stage_bytes;
        // the words of the warp's GW groups (rows pr and pr + 8, words 2q and 2q + 1 of each)
        uint2 wa[GW], wb[GW];
#pragma unroll
        for (int gi = 0; gi < GW; ++gi) {
            const int g = g0 + min(gi, max(ng - 1, 0));     // group within the chunk
            const int slab = g >> 2, wofs = (g & 3) * 8 + 2 * q;
            const uint32_t sw = (uint32_t((wofs >> 2) ^ (pr & 7)) << 4) | uint32_t((wofs & 3) * 4);
            const uint32_t base = tile + slab * kSlabTile + sw;
            wa[gi] = lds_u2(base + pr * 128);
            wb[gi] = lds_u2(base + (pr + 8) * 128);
        }
        // this lane's scales (and offsets): rows pr and pr + 8, group q of the warp's groups
        Sc cur{0, 0, 0, 0};
        const bool has_mu = kind == 0 && a.w[sg.wi].mu;
        if (q < ng) {
            const int64_t row0 = kind ? int64_t(meta[2 * k]) + int64_t(jj) * kStrip : int64_t(jj) * kStrip;
            const int skew = int((uint64_t(row0) * a.G * 2) & 15);
            const int gq = c * gcmax + g0 + q;
            const unsigned short* sc = reinterpret_cast<const unsigned short*>(sc_base + s * sc_stride + skew) + gq;
            cur.sa = sc[pr * a.G];
            cur.sb = sc[(pr + 8) * a.G];
            if (has_mu) {
                const unsigned short* m = reinterpret_cast<const unsigned short*>(mu_base + s * sc_stride + skew) + gq;
                cur.ma = m[pr * a.G];
                cur.mb = m[(pr + 8) * a.G];
            }
        }
        // the words and scales are in registers: the stage may be refilled
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        // GW independent accumulator chains, their MMAs interleaved step by step
        Pending nw;
#pragma unroll
        for (int gi = 0; gi < 4; ++gi) nw.acc[gi][0] = nw.acc[gi][1] = nw.acc[gi][2] = nw.acc[gi][3] = 0.f;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            uint32_t sh[GW][4];
#pragma unroll
            for (int gi = 0; gi < GW; ++gi) {
                const uint32_t a0 = h ? wa[gi].y : wa[gi].x, b0 = h ? wb[gi].y : wb[gi].x;
                sh[gi][0] = a0; sh[gi][1] = a0 >> 6;
                sh[gi][2] = b0; sh[gi][3] = b0 >> 6;
            }
#define TERN_D1_STEP(I)                                                                                \
    _Pragma("unroll") for (int gi = 0; gi < GW; ++gi) {                                                \
        uint32_t A[4];                                                                                 \
        decode_mma_in_place<I>(sh[gi][0], sh[gi][1], sh[gi][2], sh[gi][3], A);                         \
        mma_16816(nw.acc[gi], A, xr[8 * h + 2 * (I)], xr[8 * h + 2 * (I) + 1]);                        \
    }
            TERN_D1_STEP(0)
            TERN_D1_STEP(1)
            TERN_D1_STEP(2)
            TERN_D1_STEP(3)
#undef TERN_D1_STEP
        }
        nw.sc = cur;
        nw.s = s;
        nw.round = round;
        nw.c = c;
        nw.ng = ng;
        nw.mu = has_mu ? 1 : 0;
        if (!finish(nw)) return false;
        ++job;
        return true;
    });
}

// ------------------------------------------------------------------ host side
// plane [rows, K/16] uint32 viewed as [slab][row][32 words]: dims {32, rows, K/512}, box
// {32, 16, SB}, 128-byte swizzle.
bool slab_map(CUtensorMap* map, const uint32_t* plane, int64_t rows, int64_t K, int SB) {
    auto enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {32, cuuint64_t(rows > 0 ? rows : 1), cuuint64_t(K / 512)};
    const cuuint64_t strides[2] = {cuuint64_t(K / 4), 128};
    const cuuint32_t box[3] = {32, kStrip, cuuint32_t(SB)};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<uint32_t*>(plane), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


struct Layout {
    int W, SB, GW, nchunk, NS;
    int o_sc, o_mu, o_red, o_xs, o_cofs, o_xsum, o_meta, o_bslot, o_mainy, o_resy, o_bar, total;
};

// Consumer warps, slabs per stage and groups per warp: every warp computes GW groups per stage
// (ceil of the chunk's groups over W), so the split that wastes the fewest computed groups wins;
// W is 8 or 10 (ties: 8).
void plan_warps(int G, int& W, int& SB, int& GW) {
    double best = -1.0;
    for (int w : {8, 10}) {
        const int sb = std::min(G / 4, w);
        const int gcmax = 4 * sb, nchunk = (G + gcmax - 1) / gcmax;
        const int gw = (gcmax + w - 1) / w;
        const double eff = double(G) / (double(nchunk) * gw * w);
        if (eff > best + 1e-9) {
            best = eff;
            W = w;
            SB = sb;
            GW = gw;
        }
    }
}

bool make_layout(int K, int NSwant, Layout& L) {
    const int G = K / kGroup;
    plan_warps(G, L.W, L.SB, L.GW);
    L.nchunk = (G + 4 * L.SB - 1) / (4 * L.SB);
    auto up = [](int v, int a) { return (v + a - 1) / a * a; };
    for (int NS = NSwant; NS >= 2; --NS) {
        int o = NS * L.SB * kSlabTile;
        const int sc_stride = (32 * G + 16 + 15) & ~15;
        L.o_sc = o; o += NS * sc_stride;
        L.o_mu = o; o += NS * sc_stride;
        L.o_red = o; o += up(NS * L.W * 4 * kStrip * 4, 16);
        L.o_xs = o; o += up(K * 2, 16);
        L.o_cofs = o; o += up(L.nchunk * L.W * 4 * 4, 16);
        L.o_xsum = o; o += up(L.nchunk * L.W * 4 * 4, 16);
        L.o_meta = o; o += up(kMaxSegs * 2 * 4, 16);
        L.o_bslot = o; o += up(kMaxSegs * kSegRows * 2, 16);
        L.o_mainy = o; o += kSegRows * 4;
        L.o_resy = o; o += kSegRows * 4;
        L.o_bar = o; o += up((4 * NS + 1) * 8 + 8, 16);
        L.total = o + 1024;     // alignment slack
        L.NS = NS;
        if (L.total <= 200 * 1024) return true;
    }
    return false;
}


template <int W, int GW>
tern_status launch1(const D1Maps& maps, const D1Args& args, int grid, size_t smem, cudaStream_t stream) {
    auto kernel = decode1_kernel<W, GW>;
    static std::mutex mu;
    static bool configured[64] = {false};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return TERN_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!configured[dev]) {
            if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024) != cudaSuccess)
                return TERN_ERR_CUDA;
            configured[dev] = true;
        }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(grid), 1, 1);
    cfg.blockDim = dim3((W + kProducers + 1) * 32, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kernel, maps, args) != cudaSuccess) return TERN_ERR_CUDA;
    return TERN_OK;
}

template <int W>
tern_status launch_w(const Layout& L, const D1Maps& maps, const D1Args& args, int grid, cudaStream_t stream) {
    switch (L.GW) {
        case 1: return launch1<W, 1>(maps, args, grid, size_t(L.total), stream);
        case 2: return launch1<W, 2>(maps, args, grid, size_t(L.total), stream);
        case 3: return launch1<W, 3>(maps, args, grid, size_t(L.total), stream);
        default: return launch1<W, 4>(maps, args, grid, size_t(L.total), stream);
    }
}

}  // namespace

bool decode1_supported(const tern_weight* const* ws, int nw) {
    const int64_t K = ws[0]->K;
    if (K % 512 != 0 || K / 512 > 4096) return false;
    int64_t S = 0;
    for (int i = 0; i < nw; ++i) {
        if (ws[i]->ecount) return false;
        S += (ws[i]->N + kStrip - 1) / kStrip;
    }
    const int64_t P = std::min<int64_t>(sm_count(), S);
    const int64_t per = (S + P - 1) / P;
    // segments of one CTA: its strips in pieces of kSegStrips, plus one more per weight boundary
    if ((per + kSegStrips - 1) / kSegStrips + (nw - 1) > kMaxSegs) return false;
    Layout L;
    return make_layout(int(K), 4, L);
}

tern_status decode1_launch_group(const tern_weight* const* ws, int nw, const __half* x, __half* const* ys,
                                 const tern_weight* const* next, int nnext, cudaStream_t stream) {
    D1Maps maps;
    D1Args a = {};
    const int64_t K = ws[0]->K;
    Layout L;
    if (!make_layout(int(K), kStages, L)) return TERN_ERR_SHAPE;
    int64_t S = 0;
    bool all_static = true, has_mu = false;
    for (int i = 0; i < nw; ++i) {
        const tern_weight& w = *ws[i];
        if (!slab_map(&maps.m1[i], w.plane1, w.N, K, L.SB)) return TERN_ERR_CUDA;
        if (!slab_map(&maps.m2[i], w.r > 0 ? w.plane2 : w.plane1, w.r > 0 ? w.r : w.N, K, L.SB)) return TERN_ERR_CUDA;
        D1Weight& g = a.w[i];
        g.scale1 = reinterpret_cast<const __half*>(w.scale1);
        g.scale2 = reinterpret_cast<const __half*>(w.r > 0 ? w.scale2 : w.scale1);
        g.res_slot = w.r > 0 ? w.res_slot : nullptr;
        g.mu = reinterpret_cast<const __half*>(w.mu);
        g.y = ys[i];
        g.N = w.N;
        g.r = w.r;
        g.strip0 = int32_t(S);
        g.nstrips = int32_t((w.N + kStrip - 1) / kStrip);
        S += g.nstrips;
        all_static = all_static && (w.flags & TERN_WEIGHT_STATIC);
        has_mu = has_mu || w.mu != nullptr;
    }
    a.nw = nw;
    a.x = x;
    a.status = async_status_word();
    a.K = int32_t(K);
    a.G = int32_t(K / kGroup);
    a.SB = L.SB;
    a.nchunk = L.nchunk;
    a.NS = L.NS;
    a.S = int32_t(S);
    a.static_weights = all_static ? 1 : 0;
    a.has_mu = has_mu ? 1 : 0;
    a.o_sc = L.o_sc; a.o_mu = L.o_mu; a.o_red = L.o_red; a.o_xs = L.o_xs; a.o_cofs = L.o_cofs;
    a.o_xsum = L.o_xsum; a.o_meta = L.o_meta; a.o_bslot = L.o_bslot; a.o_mainy = L.o_mainy;
    a.o_resy = L.o_resy; a.o_bar = L.o_bar;
    const int grid = int(std::min<int64_t>(sm_count(), S));
    for (int j = 0; j < nnext; ++j) {
        const tern_weight* nx = next[j];
        const int64_t G = nx->K / kGroup, rn = nx->r;
        const void* ptr[kPfPerWeight] = {nx->plane1, nx->scale1, rn > 0 ? nx->res_slot : nullptr,
                                         rn > 0 ? nx->plane2 : nullptr, rn > 0 ? nx->scale2 : nullptr, nx->mu};
        const int64_t bytes[kPfPerWeight] = {nx->N * (nx->K / 4), nx->N * G * 2, nx->N * 4, rn * (nx->K / 4),
                                             rn * G * 2, nx->N * G * 2};
        for (int i = 0; i < kPfPerWeight; ++i) {
            const int64_t b16 = bytes[i] / 16 * 16;
            if (!ptr[i] || b16 <= 0) continue;
            a.pf_ptr[a.npf] = static_cast<const uint8_t*>(ptr[i]);
            a.pf_bytes[a.npf] = b16;
            ++a.npf;
        }
    }
    for (int i = 0; i < a.npf; ++i) a.pf_per[i] = ((a.pf_bytes[i] + grid - 1) / grid + 15) / 16 * 16;
    return L.W == 10 ? launch_w<10>(L, maps, a, grid, stream) : launch_w<8>(L, maps, a, grid, stream);
}

}  // namespace tern
