// Pieces shared by the persistent decode kernels (one token, and up to 16 tokens): the walk of a
// CTA's range of 16-row strips as segments and blocks, the copies that stage a block, and the
// bounded barrier polls. A CTA's argument struct provides nw, w[i].strip0, w[i].nstrips and Sb.
#pragma once

#include "tern_device.cuh"

namespace tern {
namespace stream {

using namespace dev;

constexpr int kStrip = 16;                 // rows per strip (the MMA's M)
constexpr int kSegStrips = 16;             // strips per segment
constexpr int kSegRows = kSegStrips * kStrip;
constexpr int kMaxSegs = 8;                // segments per CTA
constexpr int kSlabBytes = 128;            // one row of one 512-wide K slab

struct Seg {
    int wi;        // weight
    int ja, jb;    // strips [ja, jb) of the weight
};

// The next segment of the strip range [j, j1): at most kSegStrips strips of one weight.
template <typename Args>
__device__ __forceinline__ bool next_seg(const Args& a, int& j, int j1, Seg& s) {
    if (j >= j1) return false;
    int wi = 0;
#pragma unroll
    for (int i = 1; i < kMaxGemvGroup; ++i)
        if (i < a.nw && j >= a.w[i].strip0) wi = i;
    const int base = a.w[wi].strip0;
    const int jb = min(min(j1, base + a.w[wi].nstrips), j + kSegStrips);
    s.wi = wi;
    s.ja = j - base;
    s.jb = jb - base;
    j = jb;
    return true;
}

// One block: Sb (or, at the end of a segment, fewer) strips of one plane of one weight.
struct Blk {
    int kind;      // 0 main plane, 1 residual plane
    int k;         // segment index within the CTA
    Seg sg;
    int first;     // first strip: of the weight (main) or of the segment's residual slots
    int n;         // strips in the block (1..Sb)
    int64_t row0;  // first row of the plane
};

// Every role walks the same block sequence: per segment, its main blocks, then its residual
// blocks (known once the epilogue warp has published the segment metadata).
// fn(block) returns false to stop.
template <typename Args, typename Fn, typename MetaWait>
__device__ __forceinline__ void walk_blocks(const Args& a, int j0, int j1, const int* meta, MetaWait meta_wait,
                                            Fn fn) {
    int j = j0, k = 0;
    Blk bk;
    bool have_meta = false;
    while (k < kMaxSegs && next_seg(a, j, j1, bk.sg)) {
        bk.k = k;
        bk.kind = 0;
        for (int f = bk.sg.ja; f < bk.sg.jb; f += a.Sb) {
            bk.first = f;
            bk.n = min(a.Sb, bk.sg.jb - f);
            bk.row0 = int64_t(f) * kStrip;
            if (!fn(bk)) return;
        }
        if (!have_meta) {
            if (!meta_wait()) return;
            have_meta = true;
        }
        const int nrs = meta[2 * k + 1];
        bk.kind = 1;
        for (int f = 0; f < nrs; f += a.Sb) {
            bk.first = f;
            bk.n = min(a.Sb, nrs - f);
            bk.row0 = int64_t(meta[2 * k]) + int64_t(f) * kStrip;
            if (!fn(bk)) return;
        }
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

// Pause between two polls of a barrier by the warps off the critical path (producers, epilogue).
constexpr unsigned kIdlePauseNs = 64;

// Bounded wait on a barrier phase, pausing pause_ns between polls. try_wait may suspend the warp
// until the phase completes (or a hardware time limit), so a waiting warp leaves its scheduler's
// issue slots to the warps that have work (measured no slower than polling with test_wait).
__device__ __forceinline__ bool mbar_poll_addr(uint32_t addr, uint32_t parity, unsigned pause_ns) {
    uint64_t t0 = 0;
    for (uint32_t i = 0;; ++i) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(addr), "r"(parity)
            : "memory");
        if (done) return true;
        const uint64_t t = clock64();
        if (i == 0) t0 = t;
        else if (t - t0 > kWaitLimitCycles) return false;
        if (pause_ns) __nanosleep(pause_ns);
    }
}

__device__ __forceinline__ bool mbar_poll(uint64_t* bar, uint32_t parity, unsigned pause_ns) {
    return mbar_poll_addr(smem_u32(bar), parity, pause_ns);
}

__device__ __forceinline__ void mbar_arrive_addr(uint32_t addr) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(addr) : "memory");
}

__device__ __forceinline__ float sel4(int q, float a0, float a1, float a2, float a3) {
    const float lo = (q & 1) ? a1 : a0, hi = (q & 1) ? a3 : a2;
    return (q & 2) ? hi : lo;
}

// Lane rows: lane row index rr of the MMA handles strip rows pi(rr) and pi(rr) + 8, with
// pi = 0, 2, 4, 6, 1, 3, 5, 7, so that each half-warp's 8-byte reads of the 128-byte-swizzled
// tile fall in 32 distinct banks.
__device__ __forceinline__ int lane_row(int rr) { return rr < 4 ? 2 * rr : 2 * (rr - 4) + 1; }


__device__ __forceinline__ unsigned short lds_u16(uint32_t addr) {
    unsigned short v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
    return v;
}


}  // namespace stream
}  // namespace tern
