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
//  * A CTA walks its range as blocks of Sb strips (Sb = 1, 2, 4 or 8, chosen per launch from the
//    strips per CTA and K). A block streams through a ring of NS stages, each stage SB 512-wide
//    K slabs of the block's 16 Sb rows (one 3D TMA box, 128-byte swizzle, no multicast). Each of
//    the W = 8 consumer warps owns one strip of the block and a fixed share of the K groups of
//    every stage, and keeps its rows' sums in registers across the block's stages: partial sums
//    leave a warp once per block, not once per stage.
//  * Two producer warps issue the planes' boxes (a bulk or TMA copy holds its issuing thread for
//    a while, so they take every other stage each) and one more the blocks' scales (and
//    offsets), one bulk copy per block into one of two block buffers. An epilogue warp adds the
//    warps' sums of each strip in warp order and writes a row at once unless it has a residual
//    row; those rows' main sums wait in shared memory for their residual block, which adds its
//    sums and writes them (so the tail after the last block is one block's rows, not a segment's).
//  * Residual rows: since R is sorted, the residual rows of a segment are the contiguous slots
//    [s_a, s_a + span) of the residual plane; they stream as extra blocks after the segment's
//    main blocks, and each row's residual sum joins its main sum before the single rounding to
//    fp16.
//  * The signed sums run on the tensor pipe as mma.sync m16n8k16 (fp16 in, fp32 accumulate),
//    A = 16 weight rows x 16 K of decoded trits. With one token, each of a warp's (up to 4)
//    groups keeps the token in its own MMA column: lanes of row index rr = 2 g hold group g's
//    activations, so one set of 16 activation registers per lane serves all of the warp's
//    groups, and each group accumulates in its own registers, whose column 2 g alone is read
//    (the other columns multiply other groups' activations and are ignored). Lane q then holds
//    group q's sums for its two rows and scales them into its running row sums; at the end of a
//    block every lane leaves its two row sums in shared memory (no shuffles on the consumers'
//    path) and the epilogue warp adds the quad's four. The groups' MMA chains are interleaved
//    step by step with their decode.
//  * Decode is branch-free: one LOP3 writes two 2-bit codes (trits p and p+8 of a word) into
//    the mantissas of an fp16 pair (B_p + c); pairs 0-4 read the codes in place and pairs 5-7
//    after one shift of the word (tern_device.cuh); the MMA sums (B_p + 1 + t) x, and
//    C = sum (B_p + 1) x, computed once per kernel and group by the same MMA chain on the
//    constant pattern, is subtracted once per group, so a zero plane cancels bit for bit. With an
//    offset, the group sums X_g come from the same chain on an all-ones pattern.
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

#include "tern_stream.cuh"

namespace tern {
namespace {

using namespace dev;
using namespace stream;

constexpr int kMaxNW = kMaxGemvGroup;      // weights per launch
constexpr int kW = 8;                      // consumer warps
constexpr int kPlaneIssuers = 2;           // warps issuing the planes' boxes
constexpr int kScaleIssuers = 1;           // warp issuing the blocks' scales and offsets
constexpr int kProducers = kPlaneIssuers + kScaleIssuers;
constexpr int kThreads = (kW + kProducers + 1) * 32;

constexpr int kStages = 8;                 // ring stages (fewer when shared memory runs short)
constexpr int kScaleBufs = 2;              // block scale buffers
constexpr int kRedBufs = 4;                // block partial-sum buffers
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
    CUtensorMap m1[kMaxNW];   // plane1 viewed as [slab][row][32 words]: box {32, 16 Sb, SB}
    CUtensorMap m2[kMaxNW];   // plane2, the same
};

struct D1Args {
    D1Weight w[kMaxNW];
    int32_t nw;
    const __half* x;          // [K]
    unsigned int* status;
    int32_t K, G, nslab;
    int32_t Sb;               // strips per block
    int32_t SB;               // slabs per stage
    int32_t nstage;           // stages per block = ceil(nslab / SB)
    int32_t NS;               // ring stages
    int32_t S;                // strips of the launch
    int32_t static_weights;
    int32_t has_mu;
    // shared-memory offsets in bytes from the 1024-aligned base (the stages start at 0)
    int32_t o_sc, o_mu, o_red, o_xs, o_cofs, o_xsum, o_meta, o_bslot, o_rslot, o_mainy, o_bar;
    int32_t sc_stride;        // bytes of one block scale buffer (16 Sb rows x G fp16, + skew)
    // L2 prefetch of the next call's weights: each CTA takes pf_per bytes of each range
    const uint8_t* pf_ptr[kPfRanges];
    int64_t pf_bytes[kPfRanges];
    int64_t pf_per[kPfRanges];
    int32_t npf;
    // the CTAs' strip ranges [jb[b], jb[b + 1]) when balanced by their residual strips (else
    // an even split)
    int32_t balanced;
    int32_t jb[kMaxBalancedGrid + 1];
};

// A consumer warp's share of a stage of gs groups: groups [g0, g0 + ng) (wi of the wps warps of
// its strip).
__device__ __forceinline__ void warp_share(int gs, int wi, int wps, int& g0, int& ng) {
    g0 = (wi * gs) / wps;
    ng = ((wi + 1) * gs) / wps - g0;
}

// GW: groups per consumer warp per stage at most (a warp with fewer repeats its last one and
// discards the extra sums).
template <int GW>
__global__ void __launch_bounds__(kThreads, 1) decode1_kernel(const __grid_constant__ D1Maps maps,
                                                             const __grid_constant__ D1Args a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int NS = a.NS, SB = a.SB, Sb = a.Sb, nstage = a.nstage;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + a.o_bar);   // [NS] the stage's box landed
    uint64_t* empty = full + NS;                  // [NS] every consumer has its words of the stage
    uint64_t* sfull = empty + NS;                 // [kScaleBufs] the block's scales landed
    uint64_t* sempty = sfull + kScaleBufs;        // [kScaleBufs] the block's scales are no longer read
    uint64_t* redfull = sempty + kScaleBufs;      // [kRedBufs] the block's partial sums are written
    uint64_t* redempty = redfull + kRedBufs;      // [kRedBufs] ... and were read
    uint64_t* meta_bar = redempty + kRedBufs;
    int* abort_flag = reinterpret_cast<int*>(meta_bar + 1);
    const uint32_t stage0 = smem_u32(smem);
    const int slab_bytes = Sb * kStrip * kSlabBytes;             // one slab of a stage: 16 Sb rows
    const int stage_bytes = SB * slab_bytes;
    uint8_t* sc_base = smem + a.o_sc;                            // [kScaleBufs][16 Sb rows][G] (skewed)
    uint8_t* mu_base = smem + a.o_mu;                            // the same for the offsets
    float* red = reinterpret_cast<float*>(smem + a.o_red);       // [kRedBufs][W][16 rows][4 quad lanes]
    __half* xs = reinterpret_cast<__half*>(smem + a.o_xs);       // [K], pairs adjacent
    float* cofs = reinterpret_cast<float*>(smem + a.o_cofs);     // [G] C of every group
    float* xsum = reinterpret_cast<float*>(smem + a.o_xsum);     // [G] X of every group
    int* meta = reinterpret_cast<int*>(smem + a.o_meta);         // [kMaxSegs][2]: s_a, residual strips
    int16_t* bslot = reinterpret_cast<int16_t*>(smem + a.o_bslot);  // [kMaxSegs][256] row -> slot - s_a
    int16_t* rslot = reinterpret_cast<int16_t*>(smem + a.o_rslot);  // [kMaxSegs][256] slot - s_a -> row
    float* main_y = reinterpret_cast<float*>(smem + a.o_mainy);  // [256] main sums of rows with a residual

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);              // the plane's issuer (plus the box's bytes)
            mbar_init(&empty[s], kW);
        }
        for (int i = 0; i < kScaleBufs; ++i) {
            mbar_init(&sfull[i], 1);             // the scales' issuer (plus the copies' bytes)
            mbar_init(&sempty[i], kW);
        }
        for (int i = 0; i < kRedBufs; ++i) {
            mbar_init(&redfull[i], kW);
            mbar_init(&redempty[i], 1);
        }
        mbar_init(meta_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    grid_launch_dependents();

    const int P = gridDim.x, b = blockIdx.x;
    // the CTA's strips [j0, j1): the host's split balanced by residual strips when it has one, else
    // [b S / P, (b + 1) S / P) in 32-bit arithmetic (the host keeps S below 2^24 and P is at most
    // the SM count, so (b + 1) S fits; a 64-bit division here cost hundreds of cycles before the
    // first copy of every launch)
    const uint32_t uS = uint32_t(a.S), uP = uint32_t(P);
    const int j0 = a.balanced ? a.jb[b] : int(uint32_t(b) * uS / uP);
    const int j1 = a.balanced ? a.jb[b + 1] : int(uint32_t(b + 1) * uS / uP);
    volatile int* vabort = abort_flag;
    auto fail = [&]() {
        *vabort = 1;
        if (a.status) atomicOr(a.status, 1u);
    };
    auto meta_wait = [&]() -> bool {
        if (mbar_poll(meta_bar, 0, 0)) return true;
        fail();
        return false;
    };

    if (warp >= kW && warp < kW + kPlaneIssuers) {
        // ------------------------------------------------------------ plane issuers
        // warp p issues the boxes of the jobs u (block stages, in walk order) with u % 4 == p
        const int pw = warp - kW;
        if (pw == 0 && lane < a.nw) {
            prefetch_tensormap(&maps.m1[lane]);
            prefetch_tensormap(&maps.m2[lane]);
        }
        if (!a.static_weights) grid_dependency_wait();
        int job = 0, last_mine = -1, js = 0, jr = 0;     // job = jr NS + js (no division per job)
        walk_blocks(a, j0, j1, meta, meta_wait, [&](const Blk& bk) -> bool {
            if (*vabort) return false;
            const CUtensorMap* map = bk.kind ? &maps.m2[bk.sg.wi] : &maps.m1[bk.sg.wi];
            for (int t = 0; t < nstage; ++t, ++job) {
                const int s = js, round = jr;
                if (++js == NS) {
                    js = 0;
                    ++jr;
                }
                if (job % kPlaneIssuers != pw) continue;
                last_mine = job;
                if (round > 0 && !mbar_poll(&empty[s], (round - 1) & 1, kIdlePauseNs)) {
                    fail();
                    return false;
                }
                if (lane == 0) {
                    // (a box that would start outside the plane is a planning error: no copy)
                    [[maybe_unused]] const int64_t prow = bk.kind ? a.w[bk.sg.wi].r : a.w[bk.sg.wi].N;
                    const bool ok = TERN_BOUNDS(a.status, bk.row0 < prow && t * SB < a.nslab);
                    mbar_arrive_expect_tx(&full[s], ok ? uint32_t(stage_bytes) : 0u);
                    if (ok) tma_load_3d(stage0 + s * stage_bytes, map, 0, int(bk.row0), t * SB, &full[s]);
                }
            }
            return true;
        });
        // the next call's weights into L2 (a hint), then wait for the copies still in flight
        if (lane == 0 && pw == 0) {
            for (int i = 0; i < a.npf; ++i) {
                const int64_t lo = int64_t(b) * a.pf_per[i], hi = min(a.pf_bytes[i], lo + a.pf_per[i]);
                if (lo < hi) prefetch_l2_bulk(a.pf_ptr[i] + lo, uint32_t(hi - lo));
            }
        }
        for (int u = max(0, job - NS); u <= last_mine; ++u)
            if (u % kPlaneIssuers == pw && !mbar_wait(&full[u % NS], (u / NS) & 1)) break;
        return;
    }

    if (warp >= kW + kPlaneIssuers && warp < kW + kProducers) {
        // ------------------------------------------------------------ scale issuers
        // warp p issues the scales (and offsets) of the blocks v with v % 2 == p: the block's rows
        // of the [*, G] arrays are one contiguous run
        const int pw = warp - kW - kPlaneIssuers;
        if (!a.static_weights) grid_dependency_wait();
        int blk = 0, last_mine = -1;
        walk_blocks(a, j0, j1, meta, meta_wait, [&](const Blk& bk) -> bool {
            if (*vabort) return false;
            if (blk % kScaleIssuers != pw) {
                ++blk;
                return true;
            }
            last_mine = blk;
            const int nb = blk % kScaleBufs, round = blk / kScaleBufs;
            if (round > 0 && !mbar_poll(&sempty[nb], (round - 1) & 1, kIdlePauseNs)) {
                fail();
                return false;
            }
            if (lane == 0) {
                const D1Weight& Wt = a.w[bk.sg.wi];
                const int64_t nrows = bk.kind ? Wt.r : Wt.N;
                const int rows = int(max(int64_t(0), min(int64_t(bk.n * kStrip), nrows - bk.row0)));
                const __half* scale = bk.kind ? Wt.scale2 : Wt.scale1;
                const __half* mu = bk.kind == 0 ? Wt.mu : nullptr;
                const uint32_t scd = smem_u32(sc_base + nb * a.sc_stride), mud = smem_u32(mu_base + nb * a.sc_stride);
                const RowRun rs = stage_plan(scd, scale, bk.row0, rows, a.G);
                const RowRun rm = mu ? stage_plan(mud, mu, bk.row0, rows, a.G) : RowRun{0, 0};
                mbar_arrive_expect_tx(&sfull[nb], rs.bytes + rm.bytes);
                stage_issue(scd, scale, rs, &sfull[nb]);
                if (mu) stage_issue(mud, mu, rm, &sfull[nb]);
            }
            ++blk;
            return true;
        });
        for (int u = max(0, blk - kScaleBufs); u <= last_mine; ++u)
            if (u % kScaleIssuers == pw && !mbar_wait(&sfull[u % kScaleBufs], (u / kScaleBufs) & 1)) break;
        return;
    }

    if (warp == kW + kProducers) {
        // ------------------------------------------------------------ epilogue
        // segment metadata: the slots of the segment's residual rows, both ways
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
                    rslot[k * kSegRows + lr] = -1;
                }
                smin = __reduce_min_sync(0xffffffffu, smin);
                smax = __reduce_max_sync(0xffffffffu, smax);
                const int span = smax >= 0 ? min(smax - smin + 1, kSegRows) : 0;
                __syncwarp();
#pragma unroll
                for (int i = 0; i < kSegRows / 32; ++i) {
                    const int d = sl[i] - smin;
                    const bool has = sl[i] >= 0 && d < span;
                    bslot[k * kSegRows + lane + 32 * i] = int16_t(has ? d : -1);
                    if (has) rslot[k * kSegRows + d] = int16_t(lane + 32 * i);
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
        const int wps = kW / Sb;
        int blk = 0;
        // per block: row r of strip st is the sum of the strip's warps st, st + Sb, ... in warp order,
        // each the sum of its quad's lanes (lanes 0 + 1, 2 + 3, then the two). A main row without a
        // residual row is written at once; the others wait in main_y for their residual block, whose
        // slots map back to their rows, so nothing is left to write when the last block is done.
        walk_blocks(a, j0, j1, meta, [] { return true; }, [&](const Blk& bk) -> bool {
            if (*vabort) return false;
            const int nr = blk % kRedBufs, round = blk / kRedBufs;
            if (!mbar_poll(&redfull[nr], round & 1, kIdlePauseNs)) {
                fail();
                return false;
            }
            const D1Weight& Wt = a.w[bk.sg.wi];
            const int64_t n_a = int64_t(bk.sg.ja) * kStrip;
            const int d0 = bk.kind ? bk.first * kStrip : (bk.first - bk.sg.ja) * kStrip;
            for (int e = lane; e < bk.n * kStrip; e += 32) {
                const int st = e >> 4, r = e & (kStrip - 1);
                float v = 0.f;
                for (int i = 0; i < wps; ++i) {
                    const float4 c = *reinterpret_cast<const float4*>(red + ((nr * kW + st + Sb * i) * kStrip + r) * 4);
                    v += (c.x + c.y) + (c.z + c.w);
                }
                const int d = d0 + e;
                if (!TERN_BOUNDS(a.status, d < kSegRows)) continue;
                if (bk.kind == 0) {
                    if (n_a + d >= Wt.N) continue;
                    if (bslot[bk.k * kSegRows + d] < 0) Wt.y[n_a + d] = __float2half_rn(v);
                    else main_y[d] = v;
                } else {
                    const int lr = rslot[bk.k * kSegRows + d];
                    if (lr >= 0 && TERN_BOUNDS(a.status, lr < kSegRows && n_a + lr < Wt.N))
                        Wt.y[n_a + lr] = __float2half_rn(main_y[lr] + v);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&redempty[nr]);
            ++blk;
            return true;
        });
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int q = lane & 3, rr = lane >> 2;
    const int pr = lane_row(rr);
    grid_dependency_wait();
    // stage x with the two activations of each pair adjacent
    for (int i = threadIdx.x; i < a.K / 16; i += kW * 32) {
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
    asm volatile("bar.sync 1, %0;" ::"n"(kW * 32) : "memory");

    // The lane's activation registers for groups [g, g + ng) of the K axis: words 2q, 2q+1 of
    // group g + rr / 2 (group g for the lanes whose column is not read).
    uint32_t xr[16];
    auto load_x = [&](int g, int ng) {
        const int gl = (rr & 1) == 0 && (rr >> 1) < ng ? (rr >> 1) : 0;
        const uint32_t src = smem_u32(xs) + uint32_t(((g + gl) * kGroup + 32 * q) * 2);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 v = lds_u4(src + 16 * i);
            xr[4 * i] = v.x; xr[4 * i + 1] = v.y; xr[4 * i + 2] = v.z; xr[4 * i + 3] = v.w;
        }
    };
    auto load_x_at = [&](uint32_t src) {
        if (!TERN_BOUNDS(a.status, src >= smem_u32(xs) && src - smem_u32(xs) + 64 <= uint32_t(a.K * 2))) return;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 v = lds_u4(src + 16 * i);
            xr[4 * i] = v.x; xr[4 * i + 1] = v.y; xr[4 * i + 2] = v.z; xr[4 * i + 3] = v.w;
        }
    };
    // C and X of every group, four groups (one slab) per chain: the same chain as the main sums
    for (int sl = warp; sl < a.nslab; sl += kW) {
        load_x(4 * sl, 4);
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
        if (rr == 0) {     // column 2q: group 4 sl + q
            cofs[4 * sl + q] = cz[0];
            xsum[4 * sl + q] = co[0];
        }
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kW * 32) : "memory");

    // the warp's strip of every block and its share of the groups of a full and of the last stage
    const int st = warp % Sb, wps = kW / Sb, wi = warp / Sb;
    int g0f, ngf, g0l, ngl;
    warp_share(4 * SB, wi, wps, g0f, ngf);
    warp_share(4 * (a.nslab - (nstage - 1) * SB), wi, wps, g0l, ngl);
    // Per-warp constants, so that a stage costs few instructions besides the decode: the byte
    // offsets within a stage of the lane's word pair (row pr) of each of its groups, and the
    // shared-memory addresses of its activations and of its groups' C and X for stage 0.
    uint32_t offf[GW], offl[GW];
#pragma unroll
    for (int gi = 0; gi < GW; ++gi) {
        const int gf = g0f + min(gi, max(ngf - 1, 0)), gl = g0l + min(gi, max(ngl - 1, 0));
        const int wf = (gf & 3) * 8 + 2 * q, wl = (gl & 3) * 8 + 2 * q;
        offf[gi] = uint32_t((gf >> 2) * slab_bytes + (st * kStrip + pr) * kSlabBytes) +
                   ((uint32_t((wf >> 2) ^ (pr & 7)) << 4) | uint32_t((wf & 3) * 4));
        offl[gi] = uint32_t((gl >> 2) * slab_bytes + (st * kStrip + pr) * kSlabBytes) +
                   ((uint32_t((wl >> 2) ^ (pr & 7)) << 4) | uint32_t((wl & 3) * 4));
    }
    const int xgf = (rr & 1) == 0 && (rr >> 1) < ngf ? (rr >> 1) : 0;
    const int xgl = (rr & 1) == 0 && (rr >> 1) < ngl ? (rr >> 1) : 0;
    const uint32_t xsf = smem_u32(xs) + uint32_t(((g0f + xgf) * kGroup + 32 * q) * 2);
    const uint32_t xsl = smem_u32(xs) + uint32_t((((nstage - 1) * 4 * SB + g0l + xgl) * kGroup + 32 * q) * 2);
    const uint32_t xstep = uint32_t(4 * SB * kGroup * 2);      // bytes of x per stage
    const int gqf = g0f + q, gql = (nstage - 1) * 4 * SB + g0l + q;
    const bool lanef = q < ngf, lanel = q < ngl;
    const uint32_t ring_end = stage0 + uint32_t(NS * stage_bytes);
    if (nstage == 1) load_x_at(xsl);      // the same activations for every stage

    uint32_t tile = stage0;                 // the next job's stage
    uint32_t fullb = smem_u32(full), emptyb = smem_u32(empty);
    uint32_t ph = 0;
    int blk = 0;
    walk_blocks(a, j0, j1, meta, meta_wait, [&](const Blk& bk) -> bool {
        if (*vabort) return false;
        const bool active = st < bk.n;
        const int nb = blk % kScaleBufs;
        bool sc_ready = false;        // the block's scales are waited for when first needed
        const bool has_mu = bk.kind == 0 && a.w[bk.sg.wi].mu != nullptr;
        const int skew = int((uint64_t(bk.row0) * a.G * 2) & 15);
        const uint32_t sca = smem_u32(sc_base + nb * a.sc_stride + skew) + uint32_t((st * kStrip + pr) * a.G * 2);
        const uint32_t scb = sca + uint32_t(8 * a.G * 2);
        const uint32_t mud = uint32_t(a.o_mu - a.o_sc);
        [[maybe_unused]] const uint32_t sc_end = smem_u32(sc_base + (nb + 1) * a.sc_stride);   // (debug checks)
        float p0 = 0.f, p1 = 0.f;
        // one stage: its words (then the stage is released), x, the MMA chains, the scaling
        auto stage = [&](const uint32_t (&off)[GW], uint32_t xsrc, bool reload_x, int gq, bool lane_on,
                         bool work) -> bool {
            if (!mbar_poll_addr(fullb, ph, 0)) {
                fail();
                return false;
            }
            uint2 wa[GW], wb[GW];
            if (work) {
#pragma unroll
                for (int gi = 0; gi < GW; ++gi) {
                    if (TERN_BOUNDS(a.status, tile - stage0 + off[gi] + 8 * kSlabBytes + 8 <= uint32_t(NS * stage_bytes))) {
                        wa[gi] = lds_u2(tile + off[gi]);
                        wb[gi] = lds_u2(tile + off[gi] + 8 * kSlabBytes);
                    } else {
                        wa[gi] = wb[gi] = make_uint2(0u, 0u);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive_addr(emptyb);
            tile += uint32_t(stage_bytes);
            fullb += 8;
            emptyb += 8;
            if (tile == ring_end) {
                tile = stage0;
                fullb = smem_u32(full);
                emptyb = smem_u32(empty);
                ph ^= 1;
            }
            if (!work) return true;
            if (reload_x) load_x_at(xsrc);
            float acc[4][4];
#pragma unroll
            for (int gi = 0; gi < 4; ++gi) acc[gi][0] = acc[gi][1] = acc[gi][2] = acc[gi][3] = 0.f;
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
        mma_16816(acc[gi], A, xr[8 * h + 2 * (I)], xr[8 * h + 2 * (I) + 1]);                           \
    }
                TERN_D1_STEP(0)
                TERN_D1_STEP(1)
                TERN_D1_STEP(2)
                TERN_D1_STEP(3)
#undef TERN_D1_STEP
            }

            if (!sc_ready) {
                if (!mbar_poll(&sfull[nb], (blk / kScaleBufs) & 1, 0)) {
                    fail();
                    return false;
                }
                sc_ready = true;
            }
            // lane q: group q's sums for rows pr and pr + 8 (column 2q of its accumulators)
            if (lane_on && TERN_BOUNDS(a.status, gq < a.G && scb + 2 * gq + 2 <= sc_end)) {
                const float v0 = sel4(q, acc[0][0], acc[1][0], acc[2][0], acc[3][0]);
                const float v1 = sel4(q, acc[0][2], acc[1][2], acc[2][2], acc[3][2]);
                const float C = cofs[gq];
                p0 = fmaf(__half2float(__ushort_as_half(lds_u16(sca + 2 * gq))), v0 - C, p0);
                p1 = fmaf(__half2float(__ushort_as_half(lds_u16(scb + 2 * gq))), v1 - C, p1);
                if (has_mu) {
                    const float X = xsum[gq];
                    p0 = fmaf(__half2float(__ushort_as_half(lds_u16(sca + mud + 2 * gq))), X, p0);
                    p1 = fmaf(__half2float(__ushort_as_half(lds_u16(scb + mud + 2 * gq))), X, p1);
                }
            }
            return true;
        };
        const bool reload = nstage > 1;
        // one call site, so that the stage body is inlined once (the last stage takes its own
        // offsets): a shorter loop for the instruction cache, measured faster than a separate copy
#pragma unroll 1
        for (int t = 0; t < nstage; ++t) {
            const bool last = t + 1 == nstage;
            uint32_t off[GW];
#pragma unroll
            for (int gi = 0; gi < GW; ++gi) off[gi] = last ? offl[gi] : offf[gi];
            if (!stage(off, last ? xsl : xsf + uint32_t(t) * xstep, reload, last ? gql : gqf + t * 4 * SB,
                       last ? lanel : lanef, active && (last ? ngl : ngf) > 0))
                return false;
        }
        // the block's scales are no longer read (a warp with no work in the block still waits for
        // them, so that the buffer's phases stay in step)
        if (!sc_ready && !mbar_poll(&sfull[nb], (blk / kScaleBufs) & 1, 0)) {
            fail();
            return false;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sempty[nb]);
        const int nr = blk % kRedBufs, round = blk / kRedBufs;
        if (round > 0 && !mbar_poll(&redempty[nr], (round - 1) & 1, 0)) {
            fail();
            return false;
        }
        if (TERN_BOUNDS(a.status, ((nr * kW + warp) * kStrip + pr + 8) * 4 + q < kRedBufs * kW * kStrip * 4)) {
            red[((nr * kW + warp) * kStrip + pr) * 4 + q] = p0;
            red[((nr * kW + warp) * kStrip + pr + 8) * 4 + q] = p1;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&redfull[nr]);
        ++blk;
        return true;
    });
}

// ------------------------------------------------------------------ host side
// plane [rows, K/16] uint32 viewed as [slab][row][32 words]: dims {32, rows, K/512}, box
// {32, 16 Sb, SB}, 128-byte swizzle.
bool slab_map(CUtensorMap* map, const uint32_t* plane, int64_t rows, int64_t K, int Sb, int SB) {
    auto enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {32, cuuint64_t(rows > 0 ? rows : 1), cuuint64_t(K / 512)};
    const cuuint64_t strides[2] = {cuuint64_t(K / 4), 128};
    const cuuint32_t box[3] = {32, cuuint32_t(kStrip * Sb), cuuint32_t(SB)};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<uint32_t*>(plane), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct Layout {
    int Sb, SB, GW, nstage, NS, sc_stride;
    int o_sc, o_mu, o_red, o_xs, o_cofs, o_xsum, o_meta, o_bslot, o_rslot, o_mainy, o_bar, total;
};

constexpr int kSmemMax = 227 * 1024;

// Strips per block and slabs per stage. A consumer warp's time per stage grows with the groups
// it computes (GW, rounded up over the warps of its strip) plus a fixed cost per stage, and per
// block a fixed cost for the hand-off; blocks are rounded up to Sb strips, and a CTA's residual
// strips (res of them) form blocks of their own. Costs in units of one group (8 MMAs of one
// warp): about 0.7 per stage and 1.8 per block (measured).
void plan_blocks(int nslab, int64_t per, int64_t res, int& Sb, int& SB, int& GW) {
    double best = 1e30;
    Sb = 1;
    SB = 1;
    GW = 4;
    for (int sb = 1; sb <= 8; sb *= 2) {
        const int wps = kW / sb;
        for (int slabs = 1; slabs <= std::min(nslab, 8 / sb); ++slabs) {
            const int gw = (4 * slabs + wps - 1) / wps;
            if (gw > 4) continue;
            const int nst = (nslab + slabs - 1) / slabs;
            const double blocks = double((per + sb - 1) / sb) + double((res + sb - 1) / sb);
            const double cost = blocks * (nst * (gw + 0.7) + 1.8);
            if (cost < best - 1e-9) {
                best = cost;
                Sb = sb;
                SB = slabs;
                GW = gw;
            }
        }
    }
}

bool make_layout(int K, int64_t per, int64_t res, bool has_mu, Layout& L) {
    const int G = K / kGroup, nslab = K / 512;
    plan_blocks(nslab, per, res, L.Sb, L.SB, L.GW);
    L.nstage = (nslab + L.SB - 1) / L.SB;
    auto up = [](int v, int a) { return (v + a - 1) / a * a; };
    const int stage_bytes = L.Sb * L.SB * kStrip * kSlabBytes;
    L.sc_stride = up(kStrip * L.Sb * G * 2 + 16, 16);
    for (int NS = kStages; NS >= 2; --NS) {
        int o = NS * stage_bytes;
        L.o_sc = o; o += kScaleBufs * L.sc_stride;
        L.o_mu = o; o += has_mu ? kScaleBufs * L.sc_stride : 0;
        L.o_red = o; o += kRedBufs * kW * kStrip * 4 * 4;
        L.o_xs = o; o += up(K * 2, 16);
        L.o_cofs = o; o += up(G * 4, 16);
        L.o_xsum = o; o += up(G * 4, 16);
        L.o_meta = o; o += up(kMaxSegs * 2 * 4, 16);
        L.o_bslot = o; o += up(kMaxSegs * kSegRows * 2, 16);
        L.o_rslot = o; o += up(kMaxSegs * kSegRows * 2, 16);
        L.o_mainy = o; o += kSegRows * 4;
        L.o_bar = o; o += up((2 * NS + 2 * kScaleBufs + 2 * kRedBufs + 1) * 8 + 8, 16);
        L.total = o + 1024;     // alignment slack
        L.NS = NS;
        if (L.total <= kSmemMax) return true;
    }
    return false;
}

template <int GW>
tern_status launch1(const D1Maps& maps, const D1Args& args, int grid, size_t smem, cudaStream_t stream) {
    auto kernel = decode1_kernel<GW>;
    static std::mutex mu;
    static bool configured[64] = {false};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return TERN_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!configured[dev]) {
            if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemMax) != cudaSuccess)
                return TERN_ERR_CUDA;
            configured[dev] = true;
        }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(grid), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
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

// Strips of the launch, strips per CTA (the largest range) and the residual strips of such a
// range (its rows' share of the residual rows, rounded up).
void launch_strips(const tern_weight* const* ws, int nw, int64_t& S, int64_t& P, int64_t& per, int64_t& res) {
    S = 0;
    int64_t rows = 0, rrows = 0;
    for (int i = 0; i < nw; ++i) {
        S += (ws[i]->N + kStrip - 1) / kStrip;
        rows += ws[i]->N;
        rrows += ws[i]->r;
    }
    P = std::max<int64_t>(1, std::min<int64_t>(sm_count(), S));
    per = (S + P - 1) / P;
    res = rrows > 0 ? (per * kStrip * rrows / std::max<int64_t>(rows, 1) + kStrip - 1) / kStrip : 0;
}

}  // namespace

bool decode1_supported(const tern_weight* const* ws, int nw) {
    const int64_t K = ws[0]->K;
    if (K % 512 != 0 || K / 512 > 4096) return false;
    bool has_mu = false;
    for (int i = 0; i < nw; ++i) {
        if (ws[i]->ecount) return false;
        has_mu = has_mu || ws[i]->mu != nullptr;
    }
    int64_t S, P, per, res;
    launch_strips(ws, nw, S, P, per, res);
    if (S >= kMaxLaunchStrips || P > 256) return false;      // the CTA ranges' 32-bit arithmetic
    // segments of one CTA: its strips in pieces of kSegStrips, plus one more per weight boundary
    if ((per + kSegStrips - 1) / kSegStrips + (nw - 1) > kMaxSegs) return false;
    Layout L;
    return make_layout(int(K), per, res, has_mu, L);
}

int decode1_ranges(const tern_weight* const* ws, int nw, int32_t* jb, int max_ctas, int& Sb, int& nstage) {
    int64_t S, P, per, res;
    launch_strips(ws, nw, S, P, per, res);
    bool has_mu = false;
    for (int i = 0; i < nw; ++i) has_mu = has_mu || ws[i]->mu != nullptr;
    Layout L;
    if (P > max_ctas || !make_layout(int(ws[0]->K), per, res, has_mu, L)) return -1;
    Sb = L.Sb;
    nstage = L.nstage;
    if (!balanced_ranges(ws, nw, S, P, L.Sb, L.nstage, kSegStrips, kMaxSegs, jb))
        for (int64_t b = 0; b <= P; ++b) jb[b] = int32_t(uint32_t(b) * uint32_t(S) / uint32_t(P));
    return int(P);
}

tern_status decode1_launch_group(const tern_weight* const* ws, int nw, const __half* x, __half* const* ys,
                                 const tern_weight* const* next, int nnext, cudaStream_t stream) {
    D1Maps maps;
    D1Args a = {};
    const int64_t K = ws[0]->K;
    int64_t S, P, per, res;
    launch_strips(ws, nw, S, P, per, res);
    bool all_static = true, has_mu = false;
    for (int i = 0; i < nw; ++i) {
        all_static = all_static && (ws[i]->flags & TERN_WEIGHT_STATIC);
        has_mu = has_mu || ws[i]->mu != nullptr;
    }
    Layout L;
    if (!make_layout(int(K), per, res, has_mu, L)) return TERN_ERR_SHAPE;
    int64_t S0 = 0;
    for (int i = 0; i < nw; ++i) {
        const tern_weight& w = *ws[i];
        if (!slab_map(&maps.m1[i], w.plane1, w.N, K, L.Sb, L.SB)) return TERN_ERR_CUDA;
        if (!slab_map(&maps.m2[i], w.r > 0 ? w.plane2 : w.plane1, w.r > 0 ? w.r : w.N, K, L.Sb, L.SB))
            return TERN_ERR_CUDA;
        D1Weight& g = a.w[i];
        g.scale1 = reinterpret_cast<const __half*>(w.scale1);
        g.scale2 = reinterpret_cast<const __half*>(w.r > 0 ? w.scale2 : w.scale1);
        g.res_slot = w.r > 0 ? w.res_slot : nullptr;
        g.mu = reinterpret_cast<const __half*>(w.mu);
        g.y = ys[i];
        g.N = w.N;
        g.r = w.r;
        g.strip0 = int32_t(S0);
        g.nstrips = int32_t((w.N + kStrip - 1) / kStrip);
        S0 += g.nstrips;
    }
    a.nw = nw;
    a.x = x;
    a.status = async_status_word();
    a.K = int32_t(K);
    a.G = int32_t(K / kGroup);
    a.nslab = int32_t(K / 512);
    a.Sb = L.Sb;
    a.SB = L.SB;
    a.nstage = L.nstage;
    a.NS = L.NS;
    a.S = int32_t(S);
    a.static_weights = all_static ? 1 : 0;
    a.has_mu = has_mu ? 1 : 0;
    a.o_sc = L.o_sc; a.o_mu = L.o_mu; a.o_red = L.o_red; a.o_xs = L.o_xs; a.o_cofs = L.o_cofs;
    a.o_xsum = L.o_xsum; a.o_meta = L.o_meta; a.o_bslot = L.o_bslot; a.o_rslot = L.o_rslot;
    a.o_mainy = L.o_mainy; a.o_bar = L.o_bar;
    a.sc_stride = L.sc_stride;
    a.balanced = balanced_ranges(ws, nw, S, P, L.Sb, L.nstage, kSegStrips, kMaxSegs, a.jb) ? 1 : 0;
    const int grid = int(P);
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
    switch (L.GW) {
        case 1: return launch1<1>(maps, a, grid, size_t(L.total), stream);
        case 2: return launch1<2>(maps, a, grid, size_t(L.total), stream);
        case 3: return launch1<3>(maps, a, grid, size_t(L.total), stream);
        default: return launch1<4>(maps, a, grid, size_t(L.total), stream);
    }
}

}  // namespace tern
