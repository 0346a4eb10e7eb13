// Prefill GEMM (M > 16): y[M, N] = x[M, K] . W^T on tcgen05 tensor cores, W dequantised from
// the packed ternary planes straight into shared memory.
//
// The operation is that of "Post-Training Ternarization of Qwen3-4B" (arXiv 2609.01962v1),
// sections 4.3-4.5: W = s1 (.) T1, plus s2 (.) T2 on the residual rows, fp16 activations
// (section 3.1); optionally a per-group offset (W = mu + ...) and an element-level second
// plane (W += s2e T2e on its listed trits; section 4.4). At M in the thousands it is a dense
// contraction, so it runs on the tensor cores; the weights are never reconstructed in global
// memory (section 14: native kernels consume the ternary planes directly).
//
// One CTA computes a 256 (tokens) x 256 (weight rows) tile with two tcgen05.mma (kind::f16,
// M = 128, N = 256, K = 16, fp32 accumulators in TMEM columns 0-255 and 256-511) per 16
// columns of K, one per half of the tokens, both reading the same dequantised weight tile: the
// dequantisation, which bounds this kernel, is done once per 256 x 256 x 64 block of MMA work.
//  * warp 0, one thread: TMA loads of the x tile (256 x 64 fp16, 128-byte swizzle) into a
//    2-stage ring, and TMA loads of the packed codes of the tile's 256 weight rows (16 bytes
//    per row per K block) and of its residual rows into an 8-stage ring that runs ahead;
//  * warp 1, one thread: issues the MMAs and commits each stage back to the producers;
//  * warps 2-9 (256 threads, one weight row each): per 64-wide K block, read the row's 16
//    bytes of 2-bit codes from shared memory, decode them to exact fp16 s1 * t1 (two trits
//    per LOP3 into fp16 magic values, one subtract, one multiply), and store the row's 128
//    bytes in the 128-byte swizzled K-major layout the MMA reads. Rows of the residual set
//    then get RN(s1*t1 + s2*t2) with one fused multiply-add. Scales are loaded two groups
//    ahead. After the K loop the same warps read the accumulator from TMEM and write y.
//  * every wait is bounded: after about two seconds the kernel records TERN_ERR_TIMEOUT in
//    a device status word, drains its own copies and MMAs, frees TMEM and returns.
#include <mutex>

#include "tern_device.cuh"

namespace tern {
namespace {

using namespace dev;

constexpr int BM = 256;                             // tokens per CTA tile
constexpr int kUmmaM = 128;                         // tokens per MMA (two MMAs per K step)
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int kStagesA = 3;                         // x tiles (from L2: the deeper ring covers its latency)
constexpr int kStages = 2;                          // dequantised W tiles
constexpr int kStagesP = 6;                         // packed codes
constexpr int kDequantThreads = 256;
constexpr int kThreads = 64 + kDequantThreads;
constexpr int kABytes = BM * BK * 2;
constexpr int kBBytes = BN * BK * 2;
constexpr int kPBytes = BN * 16;                    // 16 bytes (64 trits) of codes per row
constexpr int kResBox = 32;                         // residual rows per TMA box
constexpr int kTmemCols = 512;                     // two 128 x 256 fp32 accumulators
constexpr unsigned kTimeoutBit = 1u;

struct GemmArgs {
    const uint32_t* plane1;
    const __half* scale1;
    const uint32_t* plane2;
    const __half* scale2;
    const int32_t* res_slot;
    const __half* mu;          // [N, G] per-group offsets, or nullptr
    const uint8_t* ecount;     // element plane: [G, N] listed trits per (group, row), or nullptr
    const int32_t* ebase;      // [G * nb + 1]
    const uint8_t* eidx;       // [nnz2] (k % 128) << 1 | (t < 0)
    const __half* escale;      // [N, G]
    int64_t nnz2;
    int64_t nb;                // ceil(N / 64)
    int64_t N, K, r, M;
    int32_t G;
    __half* y;
    unsigned int* status;
};

struct SmemLayout {
    static constexpr int a_off = 0;
    static constexpr int b_off = a_off + kStagesA * kABytes;
    static constexpr int p1_off = b_off + kStages * kBBytes;                    // [kStagesP][256][16 B]
    static constexpr int p2_off = p1_off + kStagesP * kPBytes;                  // [kStagesP][256][16 B]
    static constexpr int bar_off = p2_off + kStagesP * kPBytes;
    static constexpr int nbar = 2 * kStagesA + 2 * kStages + 2 * kStagesP + 1;
    static constexpr int tmem_off = bar_off + nbar * 8;
    static constexpr int cnt_off = tmem_off + 16;                               // 8 warp counts + total
    static constexpr int list_off = cnt_off + 48;                               // int2 [BN]
    static constexpr int bytes = list_off + BN * 8;
};
constexpr size_t kSmemBytes = SmemLayout::bytes + 1024;                          // + alignment slack
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

// ------------------------------------------------------------------ PTX helpers
// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t umma_desc_sw128(const void* p) {
    const uint64_t addr = smem_u32(p);
    return ((addr & 0x3FFFFull) >> 4) | (1ull << 16) | (uint64_t(1024 >> 4) << 32) | (1ull << 46) |
           (2ull << 61);
}

// Instruction descriptor: kind::f16, A = B = fp16, D = fp32, both K-major, M = kUmmaM, N = BN.
constexpr uint32_t kIdesc = (1u << 4) | (uint32_t(BN >> 3) << 17) | (uint32_t(kUmmaM >> 4) << 24);

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t a_desc, uint64_t b_desc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(a_desc), "l"(b_desc), "r"(kIdesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// AND of `pred` over the 256 dequantising threads (named barrier 1); every one of them must call it.
__device__ __forceinline__ bool dequant_all(bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.cta.red.and.pred q, 1, %2, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(uint32_t(pred)), "n"(kDequantThreads)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 bits_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// Eight consecutive trits (the codes in the low 16 bits of v) as four fp16x2 pairs of exact t,
// natural order: (t0, t1), (t2, t3), (t4, t5), (t6, t7). Spreading v | v << 14 puts the codes of
// trits 2j and 2j+1 at bits 4j and 16 + 4j; a LOP3 writes them into the mantissa of a power of
// two B (1024 + c, 64 + c, 4 + c), and subtracting B + 1 leaves t = c - 1 exactly.
__device__ __forceinline__ void decode8(uint32_t v, __half2 (&t)[4]) {
    const uint32_t u = v | (v << 14);
    t[0] = __hsub2(bits_h2(lop3_and_or(u, 0x00030003u, 0x64006400u)), bits_h2(0x64016401u));       // 1024 + 1
    t[1] = __hsub2(bits_h2(lop3_and_or(u, 0x00300030u, 0x54005400u)), bits_h2(0x54105410u));       // 64 + 1
    t[2] = __hsub2(bits_h2(lop3_and_or(u, 0x03000300u, 0x44004400u)), bits_h2(0x45004500u));       // 4 + 1
    t[3] = __hsub2(bits_h2(lop3_and_or(u >> 4, 0x03000300u, 0x44004400u)), bits_h2(0x45004500u));
}

// Byte offset of 16-byte chunk c (K columns 8c .. 8c+7) of row n in a 128-byte swizzled tile.
__device__ __forceinline__ uint32_t sw128_offset(int n, int c) {
    return uint32_t(n) * 128u + uint32_t((c ^ (n & 7)) << 4);
}

// kElem: the weight carries an element plane (a separate instantiation, so that the plain path
// keeps its instruction stream and registers)
template <bool kElem>
__global__ void __launch_bounds__(kThreads, 1) gemm_kernel(const __grid_constant__ CUtensorMap tmap_x,
                                                           const __grid_constant__ CUtensorMap tmap_p1,
                                                           const __grid_constant__ CUtensorMap tmap_p2,
                                                           const GemmArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* smem_a = smem + SmemLayout::a_off;
    uint8_t* smem_b = smem + SmemLayout::b_off;
    uint8_t* smem_p1 = smem + SmemLayout::p1_off;
    uint8_t* smem_p2 = smem + SmemLayout::p2_off;
    uint64_t* full_a = reinterpret_cast<uint64_t*>(smem + SmemLayout::bar_off);
    uint64_t* empty_a = full_a + kStagesA;
    uint64_t* full_b = empty_a + kStagesA;
    uint64_t* empty = full_b + kStages;                // the dequantised W stage is free again
    uint64_t* full_p = empty + kStages;
    uint64_t* empty_p = full_p + kStagesP;
    uint64_t* tmem_full = empty_p + kStagesP;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SmemLayout::tmem_off);
    int* counts = reinterpret_cast<int*>(smem + SmemLayout::cnt_off);
    int2* res_list = reinterpret_cast<int2*>(smem + SmemLayout::list_off);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n0 = int64_t(blockIdx.x) * BN;
    const int64_t m0 = int64_t(blockIdx.y) * BM;
    const int num_kb = int(a.K / BK);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStagesA; ++s) {
            mbar_init(&full_a[s], 1);
            mbar_init(&empty_a[s], 1);
        }
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full_b[s], kDequantThreads);
            mbar_init(&empty[s], 1);
        }
        for (int s = 0; s < kStagesP; ++s) {
            mbar_init(&full_p[s], 1);
            mbar_init(&empty_p[s], kDequantThreads);
        }
        mbar_init(tmem_full, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_async_smem();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    // Residual rows of this tile: (local row, slot) in row order. Their slots are contiguous
    // (R is sorted), so their codes come in with TMA boxes starting at the first slot.
    int my_slot = -1;
    unsigned res_ballot = 0;
    if (warp >= 2) {
        const int t = threadIdx.x - 64;
        const int64_t n = n0 + t;
        if (a.r > 0 && n < a.N) {
            const int s = a.res_slot[n];
            if (s >= 0 && s < a.r) my_slot = s;
        }
        res_ballot = __ballot_sync(0xffffffffu, my_slot >= 0);
        if (lane == 0) counts[warp - 2] = __popc(res_ballot);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    int n_res = 0;
    for (int w = 0; w < 8; ++w) n_res += counts[w];
    if (warp >= 2 && my_slot >= 0) {
        int base = 0;
        for (int w = 0; w < warp - 2; ++w) base += counts[w];
        const int pos = base + __popc(res_ballot & ((1u << lane) - 1u));
        res_list[pos] = make_int2(threadIdx.x - 64, my_slot);
    }
    __syncthreads();
    const int s_lo = n_res > 0 ? res_list[0].y : 0;
    const int res_boxes = (n_res + kResBox - 1) / kResBox;

    bool ok = true;
    if (warp == 0) {
        if (lane == 0) {
            int issued = 0, p_issued = 0;
            for (int kb = 0; kb < num_kb && ok; ++kb) {
                // codes run up to kStagesP blocks ahead of x
                for (; p_issued < num_kb && p_issued < kb + kStagesP && ok; ++p_issued) {
                    const int sp = p_issued % kStagesP;
                    if (p_issued >= kStagesP) ok = mbar_wait(&empty_p[sp], ((p_issued / kStagesP) - 1) & 1);
                    if (!ok) break;
                    mbar_arrive_expect_tx(&full_p[sp], uint32_t(kPBytes + res_boxes * kResBox * 16));
                    tma_load_2d(smem_p1 + sp * kPBytes, &tmap_p1, p_issued * (BK / kCodesPerWord), int(n0), &full_p[sp]);
                    for (int j = 0; j < res_boxes; ++j)
                        tma_load_2d(smem_p2 + sp * kPBytes + j * kResBox * 16, &tmap_p2,
                                    p_issued * (BK / kCodesPerWord), s_lo + j * kResBox, &full_p[sp]);
                }
                if (!ok) break;
                const int s = kb % kStagesA;
                if (kb >= kStagesA) ok = mbar_wait(&empty_a[s], ((kb / kStagesA) - 1) & 1);
                if (!ok) break;
                mbar_arrive_expect_tx(&full_a[s], kABytes);
                tma_load_2d(smem_a + s * kABytes, &tmap_x, kb * BK, int(m0), &full_a[s]);
                tma_load_2d(smem_a + s * kABytes + kABytes / 2, &tmap_x, kb * BK, int(m0) + kUmmaM, &full_a[s]);
                issued = kb + 1;
            }
            // drain: every issued copy lands before the CTA may exit
            for (int kb = issued - 1; kb >= 0 && kb >= issued - kStagesA; --kb)
                if (!mbar_wait(&full_a[kb % kStagesA], (kb / kStagesA) & 1)) ok = false;
            for (int kb = p_issued - 1; kb >= 0 && kb >= p_issued - kStagesP; --kb)
                if (!mbar_wait(&full_p[kb % kStagesP], (kb / kStagesP) & 1)) ok = false;
        }
    } else if (warp == 1) {
        if (lane == 0) {
            for (int kb = 0; kb < num_kb && ok; ++kb) {
                const int s = kb % kStages, sa = kb % kStagesA;
                ok = mbar_wait(&full_a[sa], (kb / kStagesA) & 1) && mbar_wait(&full_b[s], (kb / kStages) & 1);
                if (!ok) break;
                tc_fence_after();
                const uint8_t* as = smem_a + sa * kABytes;
                const uint8_t* bs = smem_b + s * kBBytes;
#pragma unroll
                for (int k = 0; k < BK / 16; ++k) {
                    const uint64_t bd = umma_desc_sw128(bs + 32 * k);
                    const uint32_t acc = (kb > 0 || k > 0) ? 1u : 0u;
                    umma_f16(tmem_base, umma_desc_sw128(as + 32 * k), bd, acc);
                    umma_f16(tmem_base + uint32_t(BN), umma_desc_sw128(as + kABytes / 2 + 32 * k), bd, acc);
                }
                umma_commit(&empty_a[sa]);
                umma_commit(&empty[s]);
            }
            umma_commit(tmem_full);          // also on a timeout: every issued MMA retires first
            if (!mbar_wait(tmem_full, 0)) ok = false;
        }
    } else {
        // ---------------- dequantise W into the swizzled B stages
        const int t = threadIdx.x - 64;
        const int64_t n = n0 + t;
        const bool valid = n < a.N;
        const __half* srow = a.scale1 + (valid ? n : 0) * int64_t(a.G);
        // scales of this row two groups ahead; residual items (row i = item / 8, chunk item % 8)
        // of this thread: items t and t + 256 carry their scale two groups ahead too
        // and the row's offsets, likewise (zero without an offset: the fma is then the product)
        const __half* mrow = a.mu ? a.mu + (valid ? n : 0) * int64_t(a.G) : nullptr;
        __half sq[3], mq[3];
#pragma unroll
        for (int j = 0; j < 3; ++j) {
            sq[j] = (valid && j < a.G) ? srow[j] : __float2half(0.f);
            mq[j] = (mrow && valid && j < a.G) ? mrow[j] : __float2half(0.f);
        }
        const int item0 = t, item1 = t + kDequantThreads;
        const bool has0 = item0 < n_res * 8, has1 = item1 < n_res * 8;
        const __half* s2row0 = has0 ? a.scale2 + int64_t(res_list[item0 >> 3].y) * a.G : a.scale2;
        const __half* s2row1 = has1 ? a.scale2 + int64_t(res_list[item1 >> 3].y) * a.G : a.scale2;
        __half rq0[3], rq1[3];
#pragma unroll
        for (int j = 0; j < 3; ++j) {
            rq0[j] = (has0 && j < a.G) ? s2row0[j] : __float2half(0.f);
            rq1[j] = (has1 && j < a.G) ? s2row1[j] : __float2half(0.f);
        }
        // Element plane: this row's listed trits of a group start at ebase[g, its 64-row block]
        // + the counts of the rows before it in that block (a scan over the warp, plus the
        // previous warp's total for the second warp of the block). Its count, the previous
        // warp's count at the same lane, the block base and s2e are queued two groups ahead.
        constexpr bool elem = kElem;
        const bool odd = ((t >> 5) & 1) != 0;
        const int64_t eblk = (n0 + t) / kElemBlock;
        int eq_c[3] = {0, 0, 0}, eq_p[3] = {0, 0, 0}, eq_b[3] = {0, 0, 0};
        __half eq_s[3] = {__float2half(0.f), __float2half(0.f), __float2half(0.f)};
        auto elem_load = [&](int j, int g) {
            if (!elem || g >= a.G) return;
            eq_c[j] = valid ? int(__ldg(a.ecount + int64_t(g) * a.N + n)) : 0;
            eq_p[j] = (odd && n - 32 < a.N) ? int(__ldg(a.ecount + int64_t(g) * a.N + n - 32)) : 0;
            eq_b[j] = eblk < a.nb ? __ldg(a.ebase + int64_t(g) * a.nb + eblk) : 0;   // (rows past N: none)
            eq_s[j] = valid ? a.escale[n * int64_t(a.G) + g] : __float2half(0.f);
        };
#pragma unroll
        for (int j = 0; j < 3; ++j) elem_load(j, j);
        int64_t e_pos = 0, e_end = 0;   // this row's listed trits of the current group
        for (int kb = 0; kb < num_kb; ++kb) {
            const int s = kb % kStages, sp = kb % kStagesP;
            const int g = kb / 2;
            if ((kb & 1) == 0 && kb > 0) {   // a new group: shift the scale queues, load two ahead
                sq[0] = sq[1]; sq[1] = sq[2];
                mq[0] = mq[1]; mq[1] = mq[2];
                eq_c[0] = eq_c[1]; eq_c[1] = eq_c[2];
                eq_p[0] = eq_p[1]; eq_p[1] = eq_p[2];
                eq_b[0] = eq_b[1]; eq_b[1] = eq_b[2];
                eq_s[0] = eq_s[1]; eq_s[1] = eq_s[2];
                rq0[0] = rq0[1]; rq0[1] = rq0[2];
                rq1[0] = rq1[1]; rq1[1] = rq1[2];
                const int g2 = g + 2;
                if (g2 < a.G) {
                    sq[2] = valid ? srow[g2] : __float2half(0.f);
                    if (mrow) mq[2] = valid ? mrow[g2] : __float2half(0.f);
                    elem_load(2, g2);
                    if (has0) rq0[2] = s2row0[g2];
                    if (has1) rq1[2] = s2row1[g2];
                }
            }
            if (elem && (kb & 1) == 0) {
                // the row's run of this group: every lane of the warp takes part in the scans
                const int c = min(eq_c[0], kGroup);
                int incl = c, prev = min(eq_p[0], kGroup);
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int u = __shfl_up_sync(0xffffffffu, incl, o);
                    if ((t & 31) >= o) incl += u;
                    prev += __shfl_xor_sync(0xffffffffu, prev, o);
                }
                e_pos = min(max(int64_t(eq_b[0]) + (odd ? prev : 0) + incl - c, int64_t(0)), a.nnz2);
                e_end = min(e_pos + c, a.nnz2);
            }
            // the first listed trits of this half, fetched before the wait
            uint32_t ev[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) ev[j] = (elem && e_pos + j < e_end) ? uint32_t(__ldg(a.eidx + e_pos + j)) : 0xffffu;
            // every dequantising thread takes the same decision, so the named barriers below match
            ok = dequant_all(mbar_wait(&full_p[sp], (kb / kStagesP) & 1) &&
                             (kb < kStages || mbar_wait(&empty[s], ((kb / kStages) - 1) & 1)));
            if (!ok) break;
            const uint32_t bs = smem_u32(smem_b + s * kBBytes);
            const uint4 cur = lds_u4(smem_u32(smem_p1 + sp * kPBytes + t * 16));
            const __half2 s2 = __half2half2(valid ? sq[0] : __float2half(0.f));
            const __half2 m2 = __half2half2(valid ? mq[0] : __float2half(0.f));
            const uint32_t words[4] = {cur.x, cur.y, cur.z, cur.w};
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint32_t v = (c & 1) ? (words[c >> 1] >> 16) : (words[c >> 1] & 0xFFFFu);
                __half2 tt[4];
                decode8(v, tt);
                uint4 o;
                o.x = h2_bits(__hfma2(tt[0], s2, m2));
                o.y = h2_bits(__hfma2(tt[1], s2, m2));
                o.z = h2_bits(__hfma2(tt[2], s2, m2));
                o.w = h2_bits(__hfma2(tt[3], s2, m2));
                sts_u4(bs + sw128_offset(t, c), o);
            }
            if (elem && e_pos < e_end) {
                // RN(w + s2e t2e) for this row's listed trits in this half (k % 128 in [64 h, 64 h + 64))
                const __half se = eq_s[0];
                const uint32_t lim = 64u * uint32_t((kb & 1) + 1);
                auto apply = [&](uint32_t v) {
                    const uint32_t kk = (v >> 1) & 63u;
                    const uint32_t addr = bs + sw128_offset(t, int(kk >> 3)) + (kk & 7u) * 2u;
                    unsigned short h;
                    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(h) : "r"(addr));
                    const __half w = __ushort_as_half(h);
                    const __half r = (v & 1u) ? __hsub(w, se) : __hadd(w, se);
                    asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(__half_as_ushort(r)) : "memory");
                };
                int j = 0;
                for (; j < 4 && e_pos < e_end; ++j) {
                    if ((ev[j] >> 1) >= lim) break;
                    apply(ev[j]);
                    ++e_pos;
                }
                if (j == 4)
                    while (e_pos < e_end) {
                        const uint32_t v = __ldg(a.eidx + e_pos);
                        if ((v >> 1) >= lim) break;
                        apply(v);
                        ++e_pos;
                    }
            }
            if (n_res > 0) {
                asm volatile("bar.sync 1, %0;" ::"n"(kDequantThreads) : "memory");
                for (int i = t; i < n_res * 8; i += kDequantThreads) {
                    const int row = i >> 3, c = i & 7;
                    const int2 e = res_list[row];
                    const uint32_t w2 = lds_u32(smem_u32(smem_p2 + sp * kPBytes + row * 16 + (c >> 1) * 4));
                    const __half sc2 = (i == item0) ? rq0[0] : (i == item1) ? rq1[0]
                                                                            : a.scale2[int64_t(e.y) * a.G + g];
                    const __half2 s22 = __half2half2(sc2);
                    __half2 tt[4];
                    decode8((c & 1) ? (w2 >> 16) : (w2 & 0xFFFFu), tt);
                    const uint32_t dst = bs + sw128_offset(e.x, c);
                    uint4 o = lds_u4(dst);
                    o.x = h2_bits(__hfma2(tt[0], s22, bits_h2(o.x)));
                    o.y = h2_bits(__hfma2(tt[1], s22, bits_h2(o.y)));
                    o.z = h2_bits(__hfma2(tt[2], s22, bits_h2(o.z)));
                    o.w = h2_bits(__hfma2(tt[3], s22, bits_h2(o.w)));
                    sts_u4(dst, o);
                }
            }
            fence_async_smem();
            mbar_arrive(&full_b[s]);
            mbar_arrive(&empty_p[sp]);
        }
        // ---------------- epilogue: TMEM -> fp16 y (tcgen05.ld is warp-collective: ok is made warp-uniform)
        if (ok) ok = mbar_wait(tmem_full, 0);
        ok = __all_sync(0xffffffffu, ok);
        tc_fence_after();
        if (ok) {
            const int lq = warp & 3;                         // TMEM lanes 32*lq .. 32*lq+31
            const int col0 = ((warp - 2) >> 2) * (BN / 2);   // weight rows 0..127 or 128..255
#pragma unroll 1
            for (int it = 0; it < 2 * (BN / 2) / 32; ++it) {
                const int half = it / ((BN / 2) / 32), cc = (it % ((BN / 2) / 32)) * 32;
                const int64_t m = m0 + half * kUmmaM + lq * 32 + lane;
                uint32_t r[32];
                const uint32_t taddr =
                    tmem_base + (uint32_t(lq * 32) << 16) + uint32_t(half * BN + col0 + cc);
                asm volatile(
                    "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
                    "%13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, "
                    "[%32];"
                    : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                      "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
                      "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
                      "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
                      "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                    : "r"(taddr));
                asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
                if (m < a.M) {
                    const int64_t nc = n0 + col0 + cc;
                    __half* dst = a.y + m * a.N + nc;
                    uint32_t h[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        h[j] = h2_bits(__floats2half2_rn(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1])));
                    const bool vec = (nc + 32 <= a.N) && ((reinterpret_cast<uintptr_t>(dst) & 15u) == 0);
                    if (vec) {
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            reinterpret_cast<uint4*>(dst)[j] = make_uint4(h[4 * j], h[4 * j + 1], h[4 * j + 2], h[4 * j + 3]);
                    } else {
                        for (int j = 0; j < 32 && nc + j < a.N; ++j)
                            dst[j] = __ushort_as_half(static_cast<unsigned short>((j & 1) ? (h[j >> 1] >> 16)
                                                                                          : (h[j >> 1] & 0xFFFFu)));
                    }
                }
            }
        }
    }
    __syncwarp();
    if (!ok && a.status) atomicOr(a.status, kTimeoutBit);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                     : "memory");
    }
}

// ------------------------------------------------------------------ host side
}  // namespace

size_t gemm_workspace_bytes(const tern_weight&, int64_t) { return 0; }

tern_status gemm_launch(const tern_weight& w, const __half* x, int64_t M, __half* y, void*, cudaStream_t stream) {
    if (M > (int64_t(1) << 31) - BM || w.K % BK) return TERN_ERR_SHAPE;
    const int64_t n_tiles = (w.N + BN - 1) / BN, m_tiles = (M + BM - 1) / BM;
    if (n_tiles > 0x7FFFFFFF || m_tiles > 65535) return TERN_ERR_SHAPE;
    auto enc = encode_fn();
    if (!enc) return TERN_ERR_CUDA;
    CUtensorMap map;
    const cuuint64_t dims[2] = {cuuint64_t(w.K), cuuint64_t(M)};
    const cuuint64_t strides[1] = {cuuint64_t(w.K) * sizeof(__half)};
    const cuuint32_t box[2] = {BK, kUmmaM};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<__half*>(x), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return TERN_ERR_CUDA;
    // packed codes: [rows, K/16] uint32, boxes of 4 words (one 64-wide K block) x 256 or 32 rows
    CUtensorMap map_p1, map_p2;
    auto plane_map = [&](CUtensorMap* m, const uint32_t* plane, int64_t rows, uint32_t box_rows) {
        const cuuint64_t pd[2] = {cuuint64_t(w.K / kCodesPerWord), cuuint64_t(rows > 0 ? rows : 1)};
        const cuuint64_t ps[1] = {cuuint64_t(w.K / kCodesPerWord) * 4};
        const cuuint32_t pb[2] = {BK / kCodesPerWord, box_rows};
        return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(plane), pd, ps, pb, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    };
    if (!plane_map(&map_p1, w.plane1, w.N, BN)) return TERN_ERR_CUDA;
    if (!plane_map(&map_p2, w.r > 0 ? w.plane2 : w.plane1, w.r > 0 ? w.r : w.N, kResBox)) return TERN_ERR_CUDA;
    static std::mutex mu;
    static bool configured[64] = {false};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return TERN_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!configured[dev]) {
            if (cudaFuncSetAttribute(gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     int(kSmemBytes)) != cudaSuccess ||
                cudaFuncSetAttribute(gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     int(kSmemBytes)) != cudaSuccess)
                return TERN_ERR_CUDA;
            configured[dev] = true;
        }
    }
    GemmArgs a;
    a.plane1 = w.plane1;
    a.scale1 = reinterpret_cast<const __half*>(w.scale1);
    a.plane2 = w.plane2;
    a.scale2 = reinterpret_cast<const __half*>(w.scale2);
    a.res_slot = w.r > 0 ? w.res_slot : nullptr;
    a.mu = reinterpret_cast<const __half*>(w.mu);
    a.ecount = w.ecount;
    a.ebase = w.ebase;
    a.eidx = w.eidx;
    a.escale = reinterpret_cast<const __half*>(w.escale);
    a.nnz2 = w.ecount ? w.nnz2 : 0;
    a.nb = (w.N + kElemBlock - 1) / kElemBlock;
    a.N = w.N;
    a.K = w.K;
    a.r = w.r;
    a.M = M;
    a.G = int32_t(w.K / kGroup);
    a.y = y;
    a.status = async_status_word();
    const dim3 grid{unsigned(n_tiles), unsigned(m_tiles), 1u};
    if (w.ecount)
        gemm_kernel<true><<<grid, kThreads, kSmemBytes, stream>>>(map, map_p1, map_p2, a);
    else
        gemm_kernel<false><<<grid, kThreads, kSmemBytes, stream>>>(map, map_p1, map_p2, a);
    return cudaGetLastError() == cudaSuccess ? TERN_OK : TERN_ERR_CUDA;
}

}  // namespace tern
