// Decode GEMV for 2 to 16 tokens: y[M, N] = x[M, K] . W^T with W on packed 2-bit ternary planes.
//
// What it computes is the representation of "Post-Training Ternarization of Qwen3-4B"
// (arXiv 2609.01962v1), sections 4.3-4.5: one ternary plane T1 with an fp16 scale per
// (row, 128-wide K group), a residual plane T2 with its own scales on a sorted subset R of rows,
// optionally a per-group offset mu (section 4.3's asymmetric offset); activations stay fp16
// (section 3.1). Every product t*x is exact, so the layer is a signed sum of activations
// ("Can Ternary LLMs Hit 1.58 Bits per Weight?", promptzone, "What It Is and How It Works"),
// accumulated here in fp32 and rounded to fp16 once.
//
// Design: the pipeline of the one-token kernel (tern_decode1.cu) with the tokens as MMA columns.
//  * Persistent grid, one CTA per SM, each CTA a contiguous range of 16-row strips walked as
//    blocks of Sb strips; a block streams through a ring of NS stages, each stage one or two
//    512-wide K slabs of the block's rows (3D TMA box, 128-byte swizzle, no multicast). x is
//    either resident (all tokens copied once into shared memory, in pair order, each group's
//    16-byte pieces stored transposed so that a quarter warp's loads hit eight bank groups) or,
//    when it does not fit, streamed beside each stage as a second box (64 activations x M tokens
//    x 8 slab chunks, permuted in registers). Two producer warps issue the boxes, one more the
//    blocks' scales and the segment metadata, and an epilogue warp reduces the blocks.
//  * Each of the 8 consumer warps takes one K group of every stage and two strips (four with one
//    token block) of the block, so the activations of a group (one B fragment set per 8 tokens)
//    serve every strip. A decoded A fragment (16 rows x 16 K of trits, one LOP3 per pair of
//    trits; tern_device.cuh) feeds one mma.sync m16n8k16 per 8 tokens, so the decode costs the
//    same for 2 and for 16 tokens. The call gives it 9 to 16 tokens, and 4 to 8 tokens on launches
//    of at least 10 strips per CTA; the cluster kernel of tern_gemv.cu was measured faster on the
//    other calls up to 8 tokens.
//  * Lane (rr, q) of the D fragment holds rows rr and rr+8, tokens 2q and 2q+1; it scales each
//    stage's sums by the row's group scale (after subtracting C = sum (B_p + 1) x of the group
//    and token, computed in the first block by the same MMA chain on the constant pattern, so a
//    zero plane cancels bit for bit) into running sums held across the block's stages.
//  * At the end of a block each consumer warp leaves its running sums in one of two partial-sum
//    buffers (token rows padded to an odd length) and goes on; the epilogue warp adds them per
//    (row, token) in warp order: a main row without a residual row is rounded and written at
//    once, the others wait in shared memory for their residual block (the segment's residual
//    rows are the contiguous slots [s_a, s_a + span) of the residual plane, since R is sorted),
//    which adds its sum and writes the row. The consumers meet once, after the first block.
//  * Programmatic dependent launch: the next kernel may launch at once; x is read and y written
//    only after griddepcontrol.wait. Every wait is bounded and records TERN_ERR_TIMEOUT.
#include <algorithm>
#include <mutex>

#include "tern_stream.cuh"

namespace tern {
namespace {

using namespace dev;
using namespace stream;

constexpr int kMaxNW = kMaxGemvGroup;      // weights per launch
constexpr int kW = 8;                      // consumer warps
constexpr int kPlaneIssuers = 2;
constexpr int kScaleIssuers = 1;
constexpr int kProducers = kPlaneIssuers + kScaleIssuers;
constexpr int kThreads = (kW + kProducers + 1) * 32;    // + the epilogue warp; the scale issuer also writes
                                                        // the segment metadata
// strips per consumer warp: 4 with one token block, 2 with two (the registers for both blocks'
// activations and sums); a stage then holds 2 x that many strip slabs (16 or 8 KB of plane)
__host__ __device__ constexpr int strips_per_warp(int mt) { return mt == 1 ? 4 : 2; }
constexpr int kScaleBufs = 2;
constexpr int kRedBufs = 2;                // block partial-sum buffers (consumers -> epilogue)
constexpr int kMaxStages = 6;
constexpr int kTokPad = 16;                // tokens per row of the C and X tables
constexpr int kSmemMaxM = 227 * 1024;
constexpr int kPfPerWeight = 6;
constexpr int kPfRanges = kPfPerWeight * kMaxNW;

struct DMWeight {
    const __half* scale1;     // [N, G]
    const __half* scale2;     // [r, G]
    const int32_t* res_slot;  // [N] or nullptr (r == 0)
    const __half* mu;         // [N, G] or nullptr
    __half* y;                // [M, N]
    int64_t N, r;
    int32_t strip0, nstrips;
};

struct DMMaps {
    CUtensorMap m1[kMaxNW];   // plane1 viewed as [slab][row][32 words]: box {32, 16 Sb, SB}
    CUtensorMap m2[kMaxNW];   // plane2, the same
    CUtensorMap xm;           // x viewed as [chunk of 64][token][64]: box {64, M, 8 SB}
};

struct DMArgs {
    DMWeight w[kMaxNW];
    int32_t nw;
    int32_t M;
    const __half* x;          // [M, K]
    unsigned int* status;
    int32_t K, G, nslab;
    int32_t Sb, SB, nstage, NS, S;
    int32_t has_mu;
    int32_t stage_bytes;      // plane box + x box
    int32_t sc_stride;
    int32_t o_sc, o_mu, o_red, o_cofs, o_xsum, o_meta, o_bslot, o_rslot, o_mainy, o_bar;
    int32_t o_xs;             // resident x: [M][K + 32] fp16, pair order, pieces transposed (XRES)
    int32_t static_weights;
    const uint8_t* pf_ptr[kPfRanges];
    int64_t pf_bytes[kPfRanges];
    int64_t pf_per[kPfRanges];
    int32_t npf;
    // the CTAs' strip ranges [jb[b], jb[b + 1]) when balanced by their residual strips (else
    // an even split)
    int32_t balanced;
    int32_t jb[kMaxBalancedGrid + 1];
};

// Natural-order activations (nat[8h + i] = halves 16h + 2i, 16h + 2i + 1) into the order of the
// decoded pairs (xr[8h + p] = halves 16h + p, 16h + p + 8).
__device__ __forceinline__ void pair_order(const uint32_t (&nat)[16], uint32_t (&xr)[16]) {
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int p = 0; p < 8; ++p)
            xr[8 * h + p] = prmt(nat[8 * h + p / 2], nat[8 * h + p / 2 + 4], (p & 1) ? 0x7632u : 0x5410u);
}

// MT: 8-token column blocks (1 for M <= 8, 2 for M <= 16). XRES: x is staged once per CTA in
// shared memory (all tokens, in pair order) when it fits, and the stages carry the plane alone;
// otherwise each stage carries its K range of x beside the plane.
template <int MT, bool XRES>
__global__ void __launch_bounds__(kThreads, 1) decodem_kernel(const __grid_constant__ DMMaps maps,
                                                              const __grid_constant__ DMArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int kStripsPerWarp = strips_per_warp(MT);
    const int NS = a.NS, SB = a.SB, Sb = a.Sb, nstage = a.nstage, M = a.M;
    const uint32_t plane_stage = uint32_t(Sb * SB * kStrip * kSlabBytes);   // the x box follows
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + a.o_bar);   // [NS] the stage's boxes landed
    uint64_t* empty = full + NS;                  // [NS] every consumer has read the stage
    uint64_t* sfull = empty + NS;                 // [kScaleBufs] the block's scales landed
    uint64_t* sempty = sfull + kScaleBufs;        // [kScaleBufs] the block's scales are no longer read
    uint64_t* meta_bar = sempty + kScaleBufs;
    uint64_t* cbar = meta_bar + 1;                // the consumer warps' barrier after the first block
    uint64_t* redfull = cbar + 1;                 // [kRedBufs] the block's partial sums are written
    uint64_t* redempty = redfull + kRedBufs;      // [kRedBufs] ... and were read
    int* abort_flag = reinterpret_cast<int*>(redempty + kRedBufs);
    const uint32_t stage0 = smem_u32(smem);
    const int stage_bytes = a.stage_bytes;
    const int slab_bytes = Sb * kStrip * kSlabBytes;
    uint8_t* sc_base = smem + a.o_sc;                            // [kScaleBufs][16 Sb rows][G] (skewed)
    float* red = reinterpret_cast<float*>(smem + a.o_red);       // [kRedBufs][W][strips per warp][16 rows][M + 1]
    const int Mp = M + 1;                                        // (odd: the epilogue's reads spread the banks)
    const int red_stride = kW * kStripsPerWarp * kStrip * Mp;
    float* cofs = reinterpret_cast<float*>(smem + a.o_cofs);     // [G][16 tokens]
    float* xsum = reinterpret_cast<float*>(smem + a.o_xsum);     // [G][16 tokens]
    int* meta = reinterpret_cast<int*>(smem + a.o_meta);         // [kMaxSegs][2]: s_a, residual strips
    int16_t* bslot = reinterpret_cast<int16_t*>(smem + a.o_bslot);  // [kMaxSegs][256] row -> slot - s_a
    int16_t* rslot = reinterpret_cast<int16_t*>(smem + a.o_rslot);  // [kMaxSegs][256] slot - s_a -> row
    float* main_y = reinterpret_cast<float*>(smem + a.o_mainy);  // [M][256] main sums of rows with a residual

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);              // the plane issuer (plus both boxes' bytes)
            mbar_init(&empty[s], kW);
        }
        for (int i = 0; i < kScaleBufs; ++i) {
            mbar_init(&sfull[i], 1);
            mbar_init(&sempty[i], kW);
        }
        mbar_init(meta_bar, 1);
        mbar_init(cbar, kW);
        for (int i = 0; i < kRedBufs; ++i) {
            mbar_init(&redfull[i], kW);
            mbar_init(&redempty[i], 1);
        }
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
        // ------------------------------------------------------------ plane (and x) issuers
        const int pw = warp - kW;
        if (pw == 0 && lane < a.nw) {
            prefetch_tensormap(&maps.m1[lane]);
            prefetch_tensormap(&maps.m2[lane]);
        }
        if (!XRES && pw == 0 && lane == 0) prefetch_tensormap(&maps.xm);
        // x may be written by the previous kernel; with x resident the stages hold static weights
        // only, which may stream before the wait
        if (!XRES || !a.static_weights) grid_dependency_wait();
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
                    const uint32_t dst = stage0 + s * stage_bytes;
                    [[maybe_unused]] const int64_t prow = bk.kind ? a.w[bk.sg.wi].r : a.w[bk.sg.wi].N;
                    const bool ok = TERN_BOUNDS(a.status, bk.row0 < prow && t * SB < a.nslab);
                    mbar_arrive_expect_tx(&full[s], ok ? uint32_t(stage_bytes) : 0u);
                    if (ok) {
                        tma_load_3d(dst, map, 0, int(bk.row0), t * SB, &full[s]);
                        if (!XRES) tma_load_3d(dst + plane_stage, &maps.xm, 0, 0, t * 8 * SB, &full[s]);
                    }
                }
            }
            return true;
        });
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
        // ------------------------------------------------------------ scale issuer
        // first the segment metadata: the slots of each segment's residual rows, both ways
        {
        int j = j0, k = 0;
            Seg sg;
            while (k < kMaxSegs && next_seg(a, j, j1, sg)) {
                const DMWeight& Wt = a.w[sg.wi];
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
        int blk = 0;
        int last = -1;
        walk_blocks(a, j0, j1, meta, meta_wait, [&](const Blk& bk) -> bool {
            if (*vabort) return false;
            last = blk;
            const int nb = blk % kScaleBufs, round = blk / kScaleBufs;
            if (round > 0 && !mbar_poll(&sempty[nb], (round - 1) & 1, kIdlePauseNs)) {
                fail();
                return false;
            }
            if (lane == 0) {
                const DMWeight& Wt = a.w[bk.sg.wi];
                const int64_t nrows = bk.kind ? Wt.r : Wt.N;
                const int rows = int(max(int64_t(0), min(int64_t(bk.n * kStrip), nrows - bk.row0)));
                const __half* scale = bk.kind ? Wt.scale2 : Wt.scale1;
                const __half* mu = bk.kind == 0 ? Wt.mu : nullptr;
                const uint32_t scd = smem_u32(sc_base + nb * a.sc_stride);
                const uint32_t mud = smem_u32(smem + a.o_mu + nb * a.sc_stride);
                const RowRun rs = stage_plan(scd, scale, bk.row0, rows, a.G);
                const RowRun rm = mu ? stage_plan(mud, mu, bk.row0, rows, a.G) : RowRun{0, 0};
                mbar_arrive_expect_tx(&sfull[nb], rs.bytes + rm.bytes);
                stage_issue(scd, scale, rs, &sfull[nb]);
                if (mu) stage_issue(mud, mu, rm, &sfull[nb]);
            }
            ++blk;
            return true;
        });
        for (int u = max(0, blk - kScaleBufs); u <= last; ++u)
            if (!mbar_wait(&sfull[u % kScaleBufs], (u / kScaleBufs) & 1)) break;
        return;
    }

    if (warp == kW + kProducers) {
        // ------------------------------------------------------------ epilogue
        // per block: the (row, token) sums over the strip's warps, in warp order (strip st's warps
        // are (st % ss) gs4 + g, g < gs4, each with it as its strip st / ss); a main row without a
        // residual row is written at once, the others wait in main_y for their residual block.
        // Lanes take tokens fastest (the partial sums' token rows are padded to an odd length).
        grid_dependency_wait();       // y may still be read by the previous kernel
        if (!meta_wait()) return;     // the segments' slot tables
        const int gs4 = 4 * SB, ss = kW / gs4;
        int blk = 0;
        walk_blocks(a, j0, j1, meta, meta_wait, [&](const Blk& bk) -> bool {
            if (*vabort) return false;
            const int nr = blk % kRedBufs, rround = blk / kRedBufs;
            if (!mbar_poll(&redfull[nr], rround & 1, kIdlePauseNs)) {
                fail();
                return false;
            }
            const float* redb = red + nr * red_stride;
            const DMWeight& Wt = a.w[bk.sg.wi];
            __half* yw = Wt.y;
            const int64_t Nw = Wt.N;
            const int64_t n_a = int64_t(bk.sg.ja) * kStrip;
            const int cells = bk.n * kStrip * M;
            const int gstride = kStripsPerWarp * kStrip * Mp;      // from one warp's sums to the next's
            for (int e = lane; e < cells; e += 32) {
                const int R = e / M, m = e - R * M;
                const int st = R >> 4, r = R & (kStrip - 1);
                const int w0 = (st % ss) * gs4, k = st / ss;
                const float* src = redb + ((w0 * kStripsPerWarp + k) * kStrip + r) * Mp + m;
                // gs4 is 4 or 8: all loads first, then the sum in warp order
                float t[8];
                float v;
                if (gs4 == 8) {
#pragma unroll
                    for (int g = 0; g < 8; ++g) t[g] = src[g * gstride];
                    v = 0.f;
#pragma unroll
                    for (int g = 0; g < 8; ++g) v += t[g];
                } else {
#pragma unroll
                    for (int g = 0; g < 4; ++g) t[g] = src[g * gstride];
                    v = 0.f;
#pragma unroll
                    for (int g = 0; g < 4; ++g) v += t[g];
                }
                if (bk.kind == 0) {
                    const int lr = (bk.first - bk.sg.ja) * kStrip + R;
                    if (n_a + lr < Nw && TERN_BOUNDS(a.status, lr < kSegRows)) {
                        if (bslot[bk.k * kSegRows + lr] < 0) yw[int64_t(m) * Nw + n_a + lr] = __float2half_rn(v);
                        else main_y[m * kSegRows + lr] = v;
                    }
                } else {
                    const int d = bk.first * kStrip + R;
                    const int lr = d < kSegRows ? rslot[bk.k * kSegRows + d] : -1;
                    if (lr >= 0 && TERN_BOUNDS(a.status, lr < kSegRows && n_a + lr < Nw))
                        yw[int64_t(m) * Nw + n_a + lr] = __float2half_rn(main_y[m * kSegRows + lr] + v);
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
    const int gs4 = 4 * SB;                       // groups per stage
    const int gw = warp % gs4;                    // the warp's group within a stage
    const int sw0 = warp / gs4, ss = kW / gs4;    // its strips: sw0 + ss k, k < kStripsPerWarp
    grid_dependency_wait();
    // Resident x: token rows of K + 32 halves (2K + 64 bytes: consecutive tokens 64 bytes apart
    // modulo 128), and within each group's 256 bytes the 16-byte piece i of lane q's 64 bytes
    // (q < 4, i < 4) stored at piece 4 i + q: the eight lanes of a quarter warp (two tokens, four
    // q) then read eight different 16-byte bank groups with each load
    const int xstride = a.K + 32;
    __half* xs = reinterpret_cast<__half*>(smem + a.o_xs);
    if (XRES) {
        // every token's x with the two activations of each decoded pair adjacent
        const int per_tok = a.K / 16;
        for (int u = threadIdx.x; u < M * per_tok; u += kW * 32) {
            const int m = u / per_tok, i = u - m * per_tok;
            const int g = i >> 3, uu = i & 7;         // group, and unit (pieces 2 uu, 2 uu + 1) in it
            const uint4* src = reinterpret_cast<const uint4*>(a.x + int64_t(m) * a.K + int64_t(i) * 16);
            const uint4 lo = __ldg(src), hi = __ldg(src + 1);
            uint4 o0, o1;
            o0.x = prmt(lo.x, hi.x, 0x5410u); o0.y = prmt(lo.x, hi.x, 0x7632u);
            o0.z = prmt(lo.y, hi.y, 0x5410u); o0.w = prmt(lo.y, hi.y, 0x7632u);
            o1.x = prmt(lo.z, hi.z, 0x5410u); o1.y = prmt(lo.z, hi.z, 0x7632u);
            o1.z = prmt(lo.w, hi.w, 0x5410u); o1.w = prmt(lo.w, hi.w, 0x7632u);
            uint4* grp = reinterpret_cast<uint4*>(xs + int64_t(m) * xstride + int64_t(g) * kGroup);
            const int p0 = 8 * (uu & 1) + (uu >> 1);  // piece c -> 4 (c % 4) + c / 4, c = 2 uu, 2 uu + 1
            grp[p0] = o0;
            grp[p0 + 4] = o1;
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kW * 32) : "memory");
    }

    // per-warp constants: the word offsets (row pr) of its four strips' words of its group within
    // a stage, and the x tile offsets of its group's activations for each token block
    uint32_t off[kStripsPerWarp];
#pragma unroll
    for (int k = 0; k < kStripsPerWarp; ++k) {
        const int wofs = (gw & 3) * 8 + 2 * q;
        off[k] = uint32_t((gw >> 2) * slab_bytes + ((sw0 + ss * k) * kStrip + pr) * kSlabBytes) +
                 ((uint32_t((wofs >> 2) ^ (pr & 7)) << 4) | uint32_t((wofs & 3) * 4));
    }
    // x tile row of token block o: (2 gw + q / 2) M + token; its 16-byte pieces 4 (q & 1) + i,
    // swizzled with the row
    // (resident x: token row n, lane q's pieces 4 i + q of the group, as staged above)
    uint32_t xrow[MT], xsw[MT];
#pragma unroll
    for (int o = 0; o < MT; ++o) {
        const int n = min(8 * o + rr, M - 1);
        const int row = (2 * gw + (q >> 1)) * M + n;
        xrow[o] = XRES ? smem_u32(xs) + uint32_t((n * xstride + gw * kGroup) * 2 + 16 * q) : plane_stage + uint32_t(row * 128);
        xsw[o] = uint32_t(row & 7);
    }
    const uint32_t ring_end = stage0 + uint32_t(NS * stage_bytes);
    uint32_t tile = stage0, fullb = smem_u32(full), emptyb = smem_u32(empty), ph = 0;
    // a bounded barrier of the consumer warps (a warp that gave up makes the others give up too)
    uint32_t cph = 0;
    auto csync = [&]() -> bool {
        __syncwarp();
        if (lane == 0) mbar_arrive(cbar);
        const bool ok = mbar_poll(cbar, cph, 0);
        cph ^= 1;
        if (!ok) fail();
        return ok;
    };
    int blk = 0;
    walk_blocks(a, j0, j1, meta, meta_wait, [&](const Blk& bk) -> bool {
        if (*vabort) return false;
        const int nb = blk % kScaleBufs;
        bool sc_ready = false, sc_ok = true;
        const DMWeight& Wt = a.w[bk.sg.wi];
        const bool has_mu = bk.kind == 0 && Wt.mu != nullptr;
        const int skew = int((uint64_t(bk.row0) * a.G * 2) & 15);
        const uint32_t sc0 = smem_u32(sc_base + nb * a.sc_stride + skew);
        [[maybe_unused]] const uint32_t sc_end = smem_u32(sc_base + (nb + 1) * a.sc_stride);   // (debug checks)
        const uint32_t mud = uint32_t(a.o_mu - a.o_sc);
        float run[kStripsPerWarp][MT][4];
#pragma unroll
        for (int k = 0; k < kStripsPerWarp; ++k)
#pragma unroll
            for (int o = 0; o < MT; ++o) run[k][o][0] = run[k][o][1] = run[k][o][2] = run[k][o][3] = 0.f;
        for (int t = 0; t < nstage; ++t) {
            const int gq = t * gs4 + gw;              // the warp's group of this stage
            const bool work = gq < a.G && (sw0 < bk.n);
            if (!mbar_poll_addr(fullb, ph, 0)) {
                fail();
                return false;
            }
            uint32_t xr[MT][16];
            if (work && XRES) {
                // the group's activations of stage t from the resident rows
                const uint32_t xt = uint32_t(t * gs4 * kGroup * 2);
#pragma unroll
                for (int o = 0; o < MT; ++o) {
                    if (TERN_BOUNDS(a.status, xrow[o] + xt + 64 * 3 + 16 <= smem_u32(xs) + uint32_t(M * xstride * 2))) {
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const uint4 v = lds_u4(xrow[o] + xt + 64 * i);
                            xr[o][4 * i] = v.x; xr[o][4 * i + 1] = v.y; xr[o][4 * i + 2] = v.z; xr[o][4 * i + 3] = v.w;
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i) xr[o][i] = 0u;
                    }
                }
            } else if (work) {
#pragma unroll
                for (int o = 0; o < MT; ++o) {
                    uint32_t nat[16] = {};
                    if (TERN_BOUNDS(a.status, xrow[o] + 128 <= uint32_t(stage_bytes))) {
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const uint4 v = lds_u4(tile + xrow[o] + ((uint32_t(4 * (q & 1) + i) ^ xsw[o]) << 4));
                            nat[4 * i] = v.x; nat[4 * i + 1] = v.y; nat[4 * i + 2] = v.z; nat[4 * i + 3] = v.w;
                        }
                    }
                    pair_order(nat, xr[o]);
                }
            }
            constexpr int kSpp = kStripsPerWarp;
#pragma unroll
            for (int pass = 0; pass < 1; ++pass) {
                uint2 wa[kSpp], wb[kSpp];
                if (work) {
#pragma unroll
                    for (int kk = 0; kk < kSpp; ++kk) {
                        if (TERN_BOUNDS(a.status, off[pass * kSpp + kk] + 8 * kSlabBytes + 8 <= plane_stage)) {
                            wa[kk] = lds_u2(tile + off[pass * kSpp + kk]);
                            wb[kk] = lds_u2(tile + off[pass * kSpp + kk] + 8 * kSlabBytes);
                        } else {
                            wa[kk] = wb[kk] = make_uint2(0u, 0u);
                        }
                    }
                }
                {
                    // every read of the stage is done: it may be refilled
                    __syncwarp();
                    if (lane == 0) mbar_arrive_addr(emptyb);
                }
                if (work) {
                float acc[kSpp][MT][4];
#pragma unroll
                for (int kk = 0; kk < kSpp; ++kk)
#pragma unroll
                    for (int o = 0; o < MT; ++o) acc[kk][o][0] = acc[kk][o][1] = acc[kk][o][2] = acc[kk][o][3] = 0.f;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t sh[kSpp][4];
#pragma unroll
                    for (int kk = 0; kk < kSpp; ++kk) {
                        const uint32_t a0 = h ? wa[kk].y : wa[kk].x, b0 = h ? wb[kk].y : wb[kk].x;
                        sh[kk][0] = a0; sh[kk][1] = a0 >> 6;
                        sh[kk][2] = b0; sh[kk][3] = b0 >> 6;
                    }
#define TERN_DM_STEP(I)                                                                                \
    _Pragma("unroll") for (int kk = 0; kk < kSpp; ++kk) {                                              \
        uint32_t A[4];                                                                                 \
        decode_mma_in_place<I>(sh[kk][0], sh[kk][1], sh[kk][2], sh[kk][3], A);                         \
        _Pragma("unroll") for (int o = 0; o < MT; ++o)                                                 \
            mma_16816(acc[kk][o], A, xr[o][8 * h + 2 * (I)], xr[o][8 * h + 2 * (I) + 1]);              \
    }
                    TERN_DM_STEP(0)
                    TERN_DM_STEP(1)
                    TERN_DM_STEP(2)
                    TERN_DM_STEP(3)
#undef TERN_DM_STEP
                }
                if (!sc_ready) {
                    sc_ok = mbar_poll(&sfull[nb], (blk / kScaleBufs) & 1, 0);
                    sc_ready = true;
                }
                // C (and X) of the group for tokens 8 o + 2q, 8 o + 2q + 1: in the first block from the
                // same MMA chain on the constant patterns (every row of D holds it), kept in shared
                // memory by the warps of strip 0 for the later blocks
                float2 C[MT], Xg[MT];
                if (blk == 0) {
#pragma unroll
                    for (int o = 0; o < MT; ++o) {
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
                                mma_16816(cz, Z, xr[o][8 * h + 2 * i], xr[o][8 * h + 2 * i + 1]);
                                if (a.has_mu) mma_16816(co, one, xr[o][8 * h + 2 * i], xr[o][8 * h + 2 * i + 1]);
                            }
                        C[o] = make_float2(cz[0], cz[1]);
                        Xg[o] = make_float2(co[0], co[1]);
                        if (sw0 == 0 && rr == 0) {
                            *reinterpret_cast<float2*>(cofs + gq * kTokPad + 8 * o + 2 * q) = C[o];
                            *reinterpret_cast<float2*>(xsum + gq * kTokPad + 8 * o + 2 * q) = Xg[o];
                        }
                    }
                    __syncwarp();
                } else {
#pragma unroll
                    for (int o = 0; o < MT; ++o) {
                        C[o] = *reinterpret_cast<const float2*>(cofs + gq * kTokPad + 8 * o + 2 * q);
                        Xg[o] = has_mu ? *reinterpret_cast<const float2*>(xsum + gq * kTokPad + 8 * o + 2 * q)
                                       : make_float2(0.f, 0.f);
                    }
                }
#pragma unroll
                for (int kk = 0; kk < kSpp; ++kk) {
                    const int k = pass * kSpp + kk;
                    const uint32_t ra = sc0 + uint32_t(((sw0 + ss * k) * kStrip + pr) * a.G * 2 + gq * 2);
                    const uint32_t rb = ra + uint32_t(8 * a.G * 2);
                    if (!TERN_BOUNDS(a.status, rb + 2 <= sc_end && gq < a.G)) continue;
                    const float fa = __half2float(__ushort_as_half(lds_u16(ra)));
                    const float fb = __half2float(__ushort_as_half(lds_u16(rb)));
                    float ma = 0.f, mb = 0.f;
                    if (has_mu) {
                        ma = __half2float(__ushort_as_half(lds_u16(ra + mud)));
                        mb = __half2float(__ushort_as_half(lds_u16(rb + mud)));
                    }
#pragma unroll
                    for (int o = 0; o < MT; ++o) {
                        run[k][o][0] = fmaf(fa, acc[kk][o][0] - C[o].x, run[k][o][0]);
                        run[k][o][1] = fmaf(fa, acc[kk][o][1] - C[o].y, run[k][o][1]);
                        run[k][o][2] = fmaf(fb, acc[kk][o][2] - C[o].x, run[k][o][2]);
                        run[k][o][3] = fmaf(fb, acc[kk][o][3] - C[o].y, run[k][o][3]);
                        if (has_mu) {
                            run[k][o][0] = fmaf(ma, Xg[o].x, run[k][o][0]);
                            run[k][o][1] = fmaf(ma, Xg[o].y, run[k][o][1]);
                            run[k][o][2] = fmaf(mb, Xg[o].x, run[k][o][2]);
                            run[k][o][3] = fmaf(mb, Xg[o].y, run[k][o][3]);
                        }
                    }
                }
                }
            }
            if (!sc_ok) {
                fail();
                return false;
            }
            tile += uint32_t(stage_bytes);
            fullb += 8;
            emptyb += 8;
            if (tile == ring_end) {
                tile = stage0;
                fullb = smem_u32(full);
                emptyb = smem_u32(empty);
                ph ^= 1;
            }
        }
        if (!sc_ready && !mbar_poll(&sfull[nb], (blk / kScaleBufs) & 1, 0)) {
            fail();
            return false;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sempty[nb]);
        // the warp's running sums into partial-sum buffer nr (red[nr][warp][k][row][token]), for the
        // epilogue warp; the consumers go on with the next block
        const int nr = blk % kRedBufs, rround = blk / kRedBufs;
        if (rround > 0 && !mbar_poll(&redempty[nr], (rround - 1) & 1, 0)) {
            fail();
            return false;
        }
        float* redb = red + nr * red_stride;
#pragma unroll
        for (int k = 0; k < kStripsPerWarp; ++k)
#pragma unroll
            for (int o = 0; o < MT; ++o) {
                const int n0 = 8 * o + 2 * q;
                float* ra = redb + ((warp * kStripsPerWarp + k) * kStrip + pr) * Mp;
                float* rb = ra + 8 * Mp;
                if (!TERN_BOUNDS(a.status, (warp * kStripsPerWarp + k) * kStrip + pr + 8 < kW * kStripsPerWarp * kStrip))
                    continue;
                if (n0 < M) {
                    ra[n0] = run[k][o][0];
                    rb[n0] = run[k][o][2];
                }
                if (n0 + 1 < M) {
                    ra[n0 + 1] = run[k][o][1];
                    rb[n0 + 1] = run[k][o][3];
                }
            }
        __syncwarp();
        if (lane == 0) mbar_arrive(&redfull[nr]);
        // the C and X tables of the first block are read by other warps from the second block on
        if (blk == 0 && !csync()) return false;
        ++blk;
        return true;
    });
}

// ------------------------------------------------------------------ host side
bool plane_slab_map(CUtensorMap* map, const uint32_t* plane, int64_t rows, int64_t K, int Sb, int SB) {
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

// x [M, K] fp16 viewed as [K/64 chunks][M tokens][64]: box {64, M, 8 SB} (SB slabs), 128-byte swizzle.
bool x_map(CUtensorMap* map, const __half* x, int M, int64_t K, int SB) {
    auto enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {64, cuuint64_t(M), cuuint64_t(K / 64)};
    const cuuint64_t strides[2] = {cuuint64_t(K * 2), 128};
    const cuuint32_t box[3] = {64, cuuint32_t(M), cuuint32_t(8 * SB)};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<__half*>(x), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct LayoutM {
    int Sb, SB, nstage, NS, stage_bytes, sc_stride;
    bool xres;
    int o_sc, o_mu, o_red, o_cofs, o_xsum, o_meta, o_bslot, o_rslot, o_mainy, o_xs, o_bar, total;
};

// A stage holds 2 spw strip slabs (spw strips per warp): Sb = 2 spw strips x 1 slab, or spw strips
// x 2 slabs. Both give every warp the same work per stage, so the shape with fewer padded strips
// and slabs wins (ties: the taller block, half the block ends). Then the deepest ring that fits
// (at least 3 stages).
bool make_layout_m(int K, int M, int64_t per, int64_t res, bool has_mu, LayoutM& L) {
    const int G = K / kGroup, nslab = K / 512;
    const int spw = strips_per_warp(M <= 8 ? 1 : 2);
    double best = 1e30;
    for (int slabs : {1, 2}) {
        const int sb = 2 * spw / slabs;
        const int nst = (nslab + slabs - 1) / slabs;
        const double blocks = double((per + sb - 1) / sb) + double((res + sb - 1) / sb);
        const double cost = blocks * (nst * 4.7 + 3.0);
        if (cost < best - 1e-9) {
            best = cost;
            L.Sb = sb;
            L.SB = slabs;
            L.nstage = nst;
        }
    }
    auto up = [](int v, int a) { return (v + a - 1) / a * a; };
    L.sc_stride = up(kStrip * L.Sb * G * 2 + 16, 16);
    // x resident (stages of plane alone), else x streamed with each stage; at least 3 stages
    for (int xres = 1; xres >= 0; --xres) {
        L.xres = xres == 1;
        const int plane = L.Sb * L.SB * kStrip * kSlabBytes;
        L.stage_bytes = plane + (L.xres ? 0 : M * L.SB * 1024);
        for (int NS = kMaxStages; NS >= 3; --NS) {
            int o = NS * L.stage_bytes;
            L.o_sc = o; o += kScaleBufs * L.sc_stride;
            L.o_mu = o; o += has_mu ? kScaleBufs * L.sc_stride : 0;
            L.o_red = o; o += kRedBufs * kW * spw * kStrip * (M + 1) * 4;
            L.o_cofs = o; o += up(G * kTokPad * 4, 16);
            L.o_xsum = o; o += up(G * kTokPad * 4, 16);
            L.o_meta = o; o += up(kMaxSegs * 2 * 4, 16);
            L.o_bslot = o; o += kMaxSegs * kSegRows * 2;
            L.o_rslot = o; o += kMaxSegs * kSegRows * 2;
            L.o_mainy = o; o += M * kSegRows * 4;
            L.o_xs = o; o += L.xres ? up(M * (K + 32) * 2, 16) : 0;
            L.o_bar = o; o += up((2 * NS + 2 * kScaleBufs + 2 + 2 * kRedBufs) * 8 + 8, 16);
            L.total = o + 1024;
            L.NS = NS;
            if (L.total <= kSmemMaxM) return true;
        }
    }
    return false;
}

template <int MT, bool XRES>
tern_status launch_m(const DMMaps& maps, const DMArgs& args, int grid, size_t smem, cudaStream_t stream) {
    auto kernel = decodem_kernel<MT, XRES>;
    static std::mutex mu;
    static bool configured[64] = {false};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return TERN_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!configured[dev]) {
            if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemMaxM) != cudaSuccess)
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

void strips_m(const tern_weight* const* ws, int nw, int64_t& S, int64_t& P, int64_t& per, int64_t& res) {
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

int decodem_ranges(const tern_weight* const* ws, int nw, int64_t M, int32_t* jb, int max_ctas, int& Sb,
                   int& nstage) {
    int64_t S, P, per, res;
    strips_m(ws, nw, S, P, per, res);
    bool has_mu = false;
    for (int i = 0; i < nw; ++i) has_mu = has_mu || ws[i]->mu != nullptr;
    LayoutM L;
    if (P > max_ctas || !make_layout_m(int(ws[0]->K), int(M), per, res, has_mu, L)) return -1;
    Sb = L.Sb;
    nstage = L.nstage;
    if (!balanced_ranges(ws, nw, S, P, L.Sb, L.nstage, kSegStrips, kMaxSegs, jb))
        for (int64_t b = 0; b <= P; ++b) jb[b] = int32_t(uint32_t(b) * uint32_t(S) / uint32_t(P));
    return int(P);
}

bool decodem_supported(const tern_weight* const* ws, int nw, int64_t M, const void* x) {
    const int64_t K = ws[0]->K;
    if (M < 2 || M > 16 || K % 512 != 0 || K / 512 > 4096 || !aligned16(x)) return false;
    bool has_mu = false;
    for (int i = 0; i < nw; ++i) {
        if (ws[i]->ecount) return false;
        has_mu = has_mu || ws[i]->mu != nullptr;
    }
    int64_t S, P, per, res;
    strips_m(ws, nw, S, P, per, res);
    if (S >= kMaxLaunchStrips || P > 256) return false;      // the CTA ranges' 32-bit arithmetic
    // below 9 tokens the cluster kernel is faster on launches of few strips per CTA, and at 4
    // tokens on every launch of the 8B stack (measured: this kernel wins its gate+up launch, 12
    // strips per CTA, at 8 tokens and in isolation at 4, but the stack at 4 tokens is faster with
    // the cluster kernel throughout)
    if (M < kDecodemMinM && (M < kDecodemStripsMinM || per < kDecodemMinStrips)) return false;
    if ((per + kSegStrips - 1) / kSegStrips + (nw - 1) > kMaxSegs) return false;
    LayoutM L;
    return make_layout_m(int(K), int(M), per, res, has_mu, L);
}

tern_status decodem_launch_group(const tern_weight* const* ws, int nw, const __half* x, int64_t M, __half* const* ys,
                                 const tern_weight* const* next, int nnext, cudaStream_t stream) {
    DMMaps maps;
    DMArgs a = {};
    const int64_t K = ws[0]->K;
    int64_t S, P, per, res;
    strips_m(ws, nw, S, P, per, res);
    bool has_mu = false;
    for (int i = 0; i < nw; ++i) has_mu = has_mu || ws[i]->mu != nullptr;
    LayoutM L;
    if (!make_layout_m(int(K), int(M), per, res, has_mu, L)) return TERN_ERR_SHAPE;
    int64_t S0 = 0;
    for (int i = 0; i < nw; ++i) {
        const tern_weight& w = *ws[i];
        if (!plane_slab_map(&maps.m1[i], w.plane1, w.N, K, L.Sb, L.SB)) return TERN_ERR_CUDA;
        if (!plane_slab_map(&maps.m2[i], w.r > 0 ? w.plane2 : w.plane1, w.r > 0 ? w.r : w.N, K, L.Sb, L.SB))
            return TERN_ERR_CUDA;
        DMWeight& g = a.w[i];
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
    if (!x_map(&maps.xm, x, int(M), K, L.SB)) return TERN_ERR_CUDA;
    a.nw = nw;
    a.M = int32_t(M);
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
    a.has_mu = has_mu ? 1 : 0;
    a.stage_bytes = L.stage_bytes;
    a.sc_stride = L.sc_stride;
    a.balanced = balanced_ranges(ws, nw, S, P, L.Sb, L.nstage, kSegStrips, kMaxSegs, a.jb) ? 1 : 0;
    a.o_sc = L.o_sc; a.o_mu = L.o_mu; a.o_red = L.o_red; a.o_cofs = L.o_cofs; a.o_xsum = L.o_xsum;
    a.o_meta = L.o_meta; a.o_bslot = L.o_bslot; a.o_rslot = L.o_rslot; a.o_mainy = L.o_mainy; a.o_bar = L.o_bar;
    a.o_xs = L.o_xs;
    bool all_static = true;
    for (int i = 0; i < nw; ++i) all_static = all_static && (ws[i]->flags & TERN_WEIGHT_STATIC);
    a.static_weights = all_static ? 1 : 0;
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
    if (M <= 8)
        return L.xres ? launch_m<1, true>(maps, a, grid, size_t(L.total), stream)
                      : launch_m<1, false>(maps, a, grid, size_t(L.total), stream);
    return L.xres ? launch_m<2, true>(maps, a, grid, size_t(L.total), stream)
                  : launch_m<2, false>(maps, a, grid, size_t(L.total), stream);
}

}  // namespace tern
