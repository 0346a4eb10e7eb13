// Device-side building blocks shared by the decode and prefill kernels (not installed): inline
// PTX for shared memory, mbarriers, TMA, warp MMA and programmatic dependent launch, the
// branch-free trit decode, and the host-side tensor-map encoder.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "tern_internal.cuh"

namespace tern {
namespace dev {

// Bounded waits give up after 2^32 SM clock cycles: 2-4 s at the clocks this part runs. The
// per-SM cycle counter costs a few cycles to read, unlike the global timer, so a wait whose
// first poll fails does not pay a slow timer read.
constexpr uint64_t kWaitLimitCycles = 1ull << 32;

// Bits of the sticky status word of the asynchronous kernels.
constexpr unsigned int kStatusTimeout = 1u;    // a bounded wait ran out
constexpr unsigned int kStatusBounds = 2u;     // a TERN_DEBUG bounds check failed

// TERN_BOUNDS(status, cond): in a TERN_DEBUG build, cond is checked before an access it guards; when
// it fails the status word gets kStatusBounds and the caller skips the access (no trap, no fault).
// In the release build it is `true` and costs nothing.
#ifdef TERN_DEBUG
__device__ __forceinline__ bool bounds_ok(unsigned int* status, bool cond) {
    if (!cond && status) atomicOr(status, kStatusBounds);
    return cond;
}
#define TERN_BOUNDS(status, cond) (::tern::dev::bounds_ok((status), (cond)))
#else
#define TERN_BOUNDS(status, cond) true
#endif

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t mask, uint32_t magic) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(mask), "r"(magic));   // (a & b) | c
    return d;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// D += A . B for one m16n8k16 tile, fp16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------- shared memory, explicit
__device__ __forceinline__ uint32_t lds_u32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint2 lds_u2(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}
__device__ __forceinline__ uint4 lds_u4(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ float2 lds_f2(uint32_t a) {
    float2 v;
    asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(a));
    return v;
}
__device__ __forceinline__ float lds_h2f(uint32_t a) {
    unsigned short h;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(h) : "r"(a));
    return __half2float(__ushort_as_half(h));
}
__device__ __forceinline__ void sts_u4(uint32_t a, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// ---------------------------------------------------------------- mbarriers and TMA
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}


// Bounded wait for the completion of the phase with the given parity: false after `limit` SM
// clock cycles.
__device__ __forceinline__ bool mbar_wait_for(uint64_t* bar, uint32_t parity, uint64_t limit) {
    const uint32_t addr = smem_u32(bar);
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
        else if (t - t0 > limit) return false;
    }
}

// Bounded wait with the library's limit (kWaitLimitCycles).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
    return mbar_wait_for(bar, parity, kWaitLimitCycles);
}

// 2D tiled TMA load into this CTA's shared memory, completing on `bar` (no multicast).
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- thread-block clusters
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// The float at the same shared-memory offset as `local`, in the CTA of cluster rank `cta`.
__device__ __forceinline__ float ld_dsmem_f32(const float* local, uint32_t cta) {
    const uint32_t a = smem_u32(local);
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(a), "r"(cta));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
    return v;
}

// Store a float at the same shared-memory offset as `local`, in the CTA of cluster rank `cta`.
__device__ __forceinline__ void st_dsmem_f32(const float* local, uint32_t cta, float v) {
    const uint32_t a = smem_u32(local);
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(a), "r"(cta));
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(remote), "f"(v) : "memory");
}

// Start bringing `bytes` bytes at `p` into L2 (16-byte aligned address, bytes a multiple of 16);
// a hint with no completion to wait for.
__device__ __forceinline__ void prefetch_l2_bulk(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(p)), "r"(bytes)
                 : "memory");
}

// Asynchronous store of a float to the same shared-memory offset as `local` in the CTA of cluster
// rank `cta`, completing (as 4 transaction bytes) on that CTA's mbarrier at the offset of `bar`.
__device__ __forceinline__ void st_async_f32(const float* local, uint32_t cta, float v, const uint64_t* bar) {
    uint32_t raddr, rbar;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(raddr) : "r"(smem_u32(local)), "r"(cta));
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(rbar) : "r"(smem_u32(bar)), "r"(cta));
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(raddr),
                 "r"(__float_as_uint(v)), "r"(rbar)
                 : "memory");
}

__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------- trit decode
// Pair p of a word (trits p and p+8) as fp16x2 (B_p + c_lo, B_p + c_hi), c = t + 1: one LOP3
// writes the two 2-bit codes into the mantissa of a power of two B_p.
// B_p = 16, 4, 64, 16, 4, 64, 16, 4 for p = 0..7; wl = w << 6, wr = w >> 6.
template <int P>
__device__ __forceinline__ uint32_t decode_pair(uint32_t w, uint32_t wl, uint32_t wr) {
    constexpr uint32_t kMask[3] = {0x00300030u, 0x00C000C0u, 0x03000300u};     // mantissa bits 4-5, 6-7, 8-9
    constexpr uint32_t kMagic[3] = {0x54005400u, 0x4C004C00u, 0x44004400u};    // 64, 16, 4
    if (P == 0) return lop3_and_or(wl, kMask[1], kMagic[1]);
    if (P == 1) return lop3_and_or(wl, kMask[2], kMagic[2]);
    if (P == 2) return lop3_and_or(w, kMask[0], kMagic[0]);
    if (P == 3) return lop3_and_or(w, kMask[1], kMagic[1]);
    if (P == 4) return lop3_and_or(w, kMask[2], kMagic[2]);
    if (P == 5) return lop3_and_or(wr, kMask[0], kMagic[0]);
    if (P == 6) return lop3_and_or(wr, kMask[1], kMagic[1]);
    return lop3_and_or(wr, kMask[2], kMagic[2]);
}

// The A fragments of the four MMAs of one word pair (rows rr and rr+8 of a strip):
// A[i][0..3] = pairs (2i, 2i+1) of words wa (row rr) and wb (row rr+8).
__device__ __forceinline__ void decode_word_pair(uint32_t wa, uint32_t wb, uint32_t (&A)[4][4]) {
    const uint32_t wal = wa << 6, war = wa >> 6, wbl = wb << 6, wbr = wb >> 6;
    A[0][0] = decode_pair<0>(wa, wal, war); A[0][1] = decode_pair<0>(wb, wbl, wbr);
    A[0][2] = decode_pair<1>(wa, wal, war); A[0][3] = decode_pair<1>(wb, wbl, wbr);
    A[1][0] = decode_pair<2>(wa, wal, war); A[1][1] = decode_pair<2>(wb, wbl, wbr);
    A[1][2] = decode_pair<3>(wa, wal, war); A[1][3] = decode_pair<3>(wb, wbl, wbr);
    A[2][0] = decode_pair<4>(wa, wal, war); A[2][1] = decode_pair<4>(wb, wbl, wbr);
    A[2][2] = decode_pair<5>(wa, wal, war); A[2][3] = decode_pair<5>(wb, wbl, wbr);
    A[3][0] = decode_pair<6>(wa, wal, war); A[3][1] = decode_pair<6>(wb, wbl, wbr);
    A[3][2] = decode_pair<7>(wa, wal, war); A[3][3] = decode_pair<7>(wb, wbl, wbr);
}

// The A fragment of MMA I (pairs 2I, 2I+1) of a word pair, decoded on its own so that the MMAs
// of several independent chains can be interleaved with their decode; wal/war (wbl/wbr) are the
// word shifted left/right by 6.
template <int I>
__device__ __forceinline__ void decode_mma(uint32_t wa, uint32_t wal, uint32_t war, uint32_t wb, uint32_t wbl,
                                           uint32_t wbr, uint32_t (&A)[4]) {
    A[0] = decode_pair<2 * I>(wa, wal, war);
    A[1] = decode_pair<2 * I>(wb, wbl, wbr);
    A[2] = decode_pair<2 * I + 1>(wa, wal, war);
    A[3] = decode_pair<2 * I + 1>(wb, wbl, wbr);
}

// A second decode with one shift per word instead of two: pairs 0-4 read their codes in place
// (bits 2p, 2p+1 of each half) under the bases B_p = 1024, 256, 64, 16, 4, whose fp16 ulps are
// 1, 1/4, 1/16, 1/64, 1/256, so the code lands as an integer; pairs 5-7 come from wr = w >> 6
// under 64, 16, 4. Every B_p + c stays exact in fp16, and the MMA's products with fp16
// activations stay exact in fp32.
template <int P>
__device__ __forceinline__ uint32_t decode_pair_in_place(uint32_t w, uint32_t wr) {
    if (P == 0) return lop3_and_or(w, 0x00030003u, 0x64006400u);
    if (P == 1) return lop3_and_or(w, 0x000C000Cu, 0x5C005C00u);
    if (P == 2) return lop3_and_or(w, 0x00300030u, 0x54005400u);
    if (P == 3) return lop3_and_or(w, 0x00C000C0u, 0x4C004C00u);
    if (P == 4) return lop3_and_or(w, 0x03000300u, 0x44004400u);
    if (P == 5) return lop3_and_or(wr, 0x00300030u, 0x54005400u);
    if (P == 6) return lop3_and_or(wr, 0x00C000C0u, 0x4C004C00u);
    return lop3_and_or(wr, 0x03000300u, 0x44004400u);
}

// The A fragment of MMA I (pairs 2I, 2I+1) of rows rr (word wa) and rr+8 (word wb) under the
// in-place decode; war, wbr are the words shifted right by 6.
template <int I>
__device__ __forceinline__ void decode_mma_in_place(uint32_t wa, uint32_t war, uint32_t wb, uint32_t wbr,
                                                    uint32_t (&A)[4]) {
    A[0] = decode_pair_in_place<2 * I>(wa, war);
    A[1] = decode_pair_in_place<2 * I>(wb, wbr);
    A[2] = decode_pair_in_place<2 * I + 1>(wa, war);
    A[3] = decode_pair_in_place<2 * I + 1>(wb, wbr);
}

// B_p + 1 of the in-place decode for the pairs of MMA i, as fp16x2 bits:
// 1025 = 0x6401, 257 = 0x5C04, 65 = 0x5410, 17 = 0x4C40, 5 = 0x4500.
__device__ __forceinline__ void zero_trit_pattern_in_place(int i4, uint32_t& lo, uint32_t& hi) {
    switch (i4) {
        case 0: lo = 0x64016401u; hi = 0x5C045C04u; break;   // pairs 0, 1: bases 1024, 256
        case 1: lo = 0x54105410u; hi = 0x4C404C40u; break;   // pairs 2, 3: bases 64, 16
        case 2: lo = 0x45004500u; hi = 0x54105410u; break;   // pairs 4, 5: bases 4, 64
        default: lo = 0x4C404C40u; hi = 0x45004500u; break;  // pairs 6, 7: bases 16, 4
    }
}

constexpr uint32_t kHalf2One = 0x3C003C00u;   // the fp16 pair (1, 1)

// B_p + 1 (the decoded value of trit 0) for the pairs of MMA i (pairs 2*(i%4) and 2*(i%4)+1),
// as fp16x2 bits: 17 = 0x4C40, 5 = 0x4500, 65 = 0x5410.
__device__ __forceinline__ void zero_trit_pattern(int i4, uint32_t& lo, uint32_t& hi) {
    switch (i4) {
        case 0: lo = 0x4C404C40u; hi = 0x45004500u; break;   // pairs 0, 1: bases 16, 4
        case 1: lo = 0x54105410u; hi = 0x4C404C40u; break;   // pairs 2, 3: bases 64, 16
        case 2: lo = 0x45004500u; hi = 0x54105410u; break;   // pairs 4, 5: bases 4, 64
        default: lo = 0x4C404C40u; hi = 0x45004500u; break;  // pairs 6, 7: bases 16, 4
    }
}

// ---------------------------------------------------------------- host: tensor maps
inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2D map over an exec plane [rows, K/16] uint32: boxes of box_words x box_rows, with the
// given swizzle (128-byte swizzle needs box_words = 32).
inline bool plane_map(CUtensorMap* map, const uint32_t* plane, int64_t rows, int64_t K, uint32_t box_words,
                      uint32_t box_rows, CUtensorMapSwizzle swizzle) {
    auto enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {cuuint64_t(K / kCodesPerWord), cuuint64_t(rows > 0 ? rows : 1)};
    const cuuint64_t strides[1] = {cuuint64_t(K / kCodesPerWord) * 4};
    const cuuint32_t box[2] = {box_words, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(plane), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace dev
}  // namespace tern
