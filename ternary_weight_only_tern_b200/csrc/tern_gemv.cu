// Decode GEMV for M <= 16: y[M, N] = x[M, K] . W^T with W on packed 2-bit ternary planes.
//
// What it computes is the representation of "Post-Training Ternarization of Qwen3-4B"
// (arXiv 2609.01962v1), sections 4.3-4.5: one ternary plane T1 with an fp16 scale per
// (row, 128-wide K group), plus a residual plane T2 with its own scales on a subset R of
// rows; activations stay fp16 (section 3.1). With t in {-1, 0, +1} every product t*x is
// exact, so the layer is a signed sum of activations ("Can Ternary LLMs Hit 1.58 Bits per
// Weight?", promptzone, "What It Is and How It Works"), accumulated here in fp32.
//
// Design (B200, memory-bound at 0.266 bytes per weight):
//  * One CTA = 4 warps = 64 output rows (one 16-row strip per warp) x one K-slice. The
//    K-slices of a row block form a thread-block cluster; partial sums are reduced over
//    distributed shared memory in a fixed order (no global workspace, no atomics, no
//    spin-waits), and the CTA of rank c writes rows [c*64/S, (c+1)*64/S) of the block.
//  * The signed sums run on the tensor pipe as mma.sync m16n8k16 (fp16 in, fp32
//    accumulate): A = 16 weight rows x 16 K of decoded trits, B = the activations of up to
//    8 tokens. The products are exact (+-x or 0), so this is the fp32-accumulated
//    add/subtract of the method, with the decode cost independent of M.
//  * Decode is branch-free: one LOP3 turns two 2-bit codes (bits p and p+16 of a word) into
//    an fp16 pair (B_p + c) by writing the code into the mantissa of a power of two B_p; a
//    shift by 6 either way moves the codes of bits 0-3 and 10-15 into mantissa positions,
//    so a word of 16 trits costs 2 shifts and 8 LOP3. Since c = t + 1, the MMA then sums
//    (B_p + 1 + t) * x from zero, and C = sum (B_p + 1) * x is subtracted once per group. C is
//    computed once per CTA by the same MMA on the constant pattern B_p + 1 in the same K
//    order, so a zero plane cancels bit for bit. The bases are 4, 16 and 64, so the offsets
//    are small and every partial sum is exact on integer inputs. A non-finite activation
//    makes every output of its token non-finite (NaN where the dense product has +-inf).
//  * The contraction order over K is free, so the MMA's K order follows the packed words
//    (pair j = trits j and j+8 of a word); the activations of the slice are staged in
//    shared memory in that order once per CTA.
//  * Rows of the residual plane T2 run as a first pass of the same kernel that writes fp32
//    sums to the workspace; the main pass adds them to the rows of R before its single
//    rounding to fp16.
#include <stdlib.h>

#include <algorithm>
#include <mutex>

#include "tern_internal.cuh"

namespace tern {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kRowsPerCta = 16 * kWarps;
constexpr int kMaxSplit = 16;
constexpr int kPrefetch = 4;                  // groups of packed words in flight per warp
constexpr int kSmemBudget = 96 * 1024;        // activations staged per CTA (bytes)
constexpr int kNegcStride = 16;               // floats per group (one per token)

struct GemvArgs {
    const uint32_t* plane;     // [rows, K/16]
    const __half* scale;       // [rows, G]
    const __half* x;           // [M, K]
    int64_t rows;
    int64_t K;
    int32_t G;
    int32_t M;
    int32_t gpc;               // groups per K-slice
    int32_t split;             // K-slices (= cluster size along x)
    __half* y;                 // main pass: [M, rows]
    float* res_out;            // residual pass: [M, rows] fp32 sums
    const float* res_in;       // main pass: [M, r] residual sums, or nullptr
    const int32_t* res_slot;   // main pass: [rows] slot map, or nullptr
    int64_t r;
};

// ------------------------------------------------------------------ PTX helpers
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

__device__ __forceinline__ uint2 ld_stream_u2(const uint32_t* p) {
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}

__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ float ld_dsmem_f32(const float* local, uint32_t cta) {
    const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(local));
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(a), "r"(cta));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
    return v;
}

// Pair p of a word (trits p and p+8) as fp16x2 (B_p + c_lo, B_p + c_hi), c = t + 1.
// B_p = 16, 4, 64, 16, 4, 64, 16, 4 for p = 0..7. wl = w << 6, wr = w >> 6.
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

// ------------------------------------------------------------------ the kernel
template <int NT, bool kResidualPass>
__global__ void __launch_bounds__(kThreads) gemv_kernel(const GemvArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int M = a.M;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int q = lane & 3, rr = lane >> 2;
    const int ks = blockIdx.x;
    const int g_begin = ks * a.gpc;
    const int ng = max(0, min(a.G, g_begin + a.gpc) - g_begin);
    const int xs_stride = a.gpc * kGroup;                     // halves per token row in smem
    __half* xs = reinterpret_cast<__half*>(smem);
    float* cofs = reinterpret_cast<float*>(smem + size_t(M) * xs_stride * sizeof(__half));
    float* red = cofs + size_t(a.gpc) * kNegcStride;          // [kRowsPerCta][16]

    // 1. Stage this slice of x, pairing columns (j, j+8) of every 16-column block.
    {
        const int blocks16 = ng * kWordsPerGroup;
        for (int idx = threadIdx.x; idx < M * blocks16; idx += kThreads) {
            const int m = idx / blocks16, b = idx - m * blocks16;
            const uint4* src =
                reinterpret_cast<const uint4*>(a.x + int64_t(m) * a.K + int64_t(g_begin) * kGroup + b * 16);
            const uint4 lo = __ldg(src), hi = __ldg(src + 1);
            uint4 o0, o1;
            o0.x = prmt(lo.x, hi.x, 0x5410u); o0.y = prmt(lo.x, hi.x, 0x7632u);
            o0.z = prmt(lo.y, hi.y, 0x5410u); o0.w = prmt(lo.y, hi.y, 0x7632u);
            o1.x = prmt(lo.z, hi.z, 0x5410u); o1.y = prmt(lo.z, hi.z, 0x7632u);
            o1.z = prmt(lo.w, hi.w, 0x5410u); o1.w = prmt(lo.w, hi.w, 0x7632u);
            uint4* dst = reinterpret_cast<uint4*>(xs + size_t(m) * xs_stride + b * 16);
            dst[0] = o0;
            dst[1] = o1;
        }
    }
    __syncthreads();

    // B fragment of MMA i in group gi for token tile t: pairs (j, j+1) of word 2q + i/4.
    auto load_b = [&](int gi, int i, int t, uint32_t& b0, uint32_t& b1) {
        const int n = 8 * t + rr;
        if (n < M) {
            const int off = gi * kGroup + 16 * (2 * q + (i >> 2)) + 4 * (i & 3);
            const uint2 v = *reinterpret_cast<const uint2*>(xs + size_t(n) * xs_stride + off);
            b0 = v.x;
            b1 = v.y;
        } else {
            b0 = 0u;
            b1 = 0u;
        }
    };

    // 2. C[g][token] = sum_k (B_p(k) + 1) * x[token][k], one MMA chain per group.
    for (int gi = warp; gi < ng; gi += kWarps) {
        float c[NT][4];
#pragma unroll
        for (int t = 0; t < NT; ++t) c[t][0] = c[t][1] = c[t][2] = c[t][3] = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            uint32_t A[4];
            zero_trit_pattern(i & 3, A[0], A[2]);
            A[1] = A[0];
            A[3] = A[2];
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                uint32_t b0, b1;
                load_b(gi, i, t, b0, b1);
                mma_16816(c[t], A, b0, b1);
            }
        }
        if (rr == 0) {
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                cofs[gi * kNegcStride + 8 * t + 2 * q] = c[t][0];
                cofs[gi * kNegcStride + 8 * t + 2 * q + 1] = c[t][1];
            }
        }
    }
    __syncthreads();

    // 3. Stream this warp's 16-row strip over the slice.
    const int64_t block_row0 = int64_t(blockIdx.y) * kRowsPerCta;
    const int64_t ra = block_row0 + warp * 16 + rr, rb = ra + 8;
    const bool va = ra < a.rows, vb = rb < a.rows;
    const int64_t wpr = a.K / kCodesPerWord;
    const uint32_t* pa = a.plane + (va ? ra : 0) * wpr + int64_t(g_begin) * kWordsPerGroup + 2 * q;
    const uint32_t* pb = a.plane + (vb ? rb : 0) * wpr + int64_t(g_begin) * kWordsPerGroup + 2 * q;
    const __half* sa_ptr = a.scale + (va ? ra : 0) * int64_t(a.G) + g_begin;
    const __half* sb_ptr = a.scale + (vb ? rb : 0) * int64_t(a.G) + g_begin;
    constexpr uint32_t kZeroCodes = 0x55555555u;                 // code 1 = trit 0 everywhere

    float yacc[NT][4];
#pragma unroll
    for (int t = 0; t < NT; ++t) yacc[t][0] = yacc[t][1] = yacc[t][2] = yacc[t][3] = 0.f;

    uint2 bufA[kPrefetch], bufB[kPrefetch];
    float bsa[kPrefetch], bsb[kPrefetch];
    auto fetch = [&](int gi, int u) {
        if (gi < ng) {
            bufA[u] = va ? ld_stream_u2(pa + gi * kWordsPerGroup) : make_uint2(kZeroCodes, kZeroCodes);
            bufB[u] = vb ? ld_stream_u2(pb + gi * kWordsPerGroup) : make_uint2(kZeroCodes, kZeroCodes);
            bsa[u] = va ? __half2float(sa_ptr[gi]) : 0.f;
            bsb[u] = vb ? __half2float(sb_ptr[gi]) : 0.f;
        }
    };
#pragma unroll
    for (int u = 0; u < kPrefetch; ++u) fetch(u, u);

    for (int base = 0; base < ng; base += kPrefetch) {
        uint2 cA[kPrefetch], cB[kPrefetch];
        float csa[kPrefetch], csb[kPrefetch];
#pragma unroll
        for (int u = 0; u < kPrefetch; ++u) {
            cA[u] = bufA[u]; cB[u] = bufB[u]; csa[u] = bsa[u]; csb[u] = bsb[u];
        }
#pragma unroll
        for (int u = 0; u < kPrefetch; ++u) fetch(base + kPrefetch + u, u);
#pragma unroll
        for (int u = 0; u < kPrefetch; ++u) {
            const int gi = base + u;
            if (gi >= ng) break;
            float acc[NT][4];
#pragma unroll
            for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t wa = h ? cA[u].y : cA[u].x, wb = h ? cB[u].y : cB[u].x;
                const uint32_t wal = wa << 6, war = wa >> 6, wbl = wb << 6, wbr = wb >> 6;
                uint32_t A[4][4];   // four MMAs per word: pairs (0,1), (2,3), (4,5), (6,7)
                A[0][0] = decode_pair<0>(wa, wal, war); A[0][1] = decode_pair<0>(wb, wbl, wbr);
                A[0][2] = decode_pair<1>(wa, wal, war); A[0][3] = decode_pair<1>(wb, wbl, wbr);
                A[1][0] = decode_pair<2>(wa, wal, war); A[1][1] = decode_pair<2>(wb, wbl, wbr);
                A[1][2] = decode_pair<3>(wa, wal, war); A[1][3] = decode_pair<3>(wb, wbl, wbr);
                A[2][0] = decode_pair<4>(wa, wal, war); A[2][1] = decode_pair<4>(wb, wbl, wbr);
                A[2][2] = decode_pair<5>(wa, wal, war); A[2][3] = decode_pair<5>(wb, wbl, wbr);
                A[3][0] = decode_pair<6>(wa, wal, war); A[3][1] = decode_pair<6>(wb, wbl, wbr);
                A[3][2] = decode_pair<7>(wa, wal, war); A[3][3] = decode_pair<7>(wb, wbl, wbr);
#pragma unroll
                for (int i4 = 0; i4 < 4; ++i4) {
#pragma unroll
                    for (int t = 0; t < NT; ++t) {
                        uint32_t b0, b1;
                        load_b(gi, 4 * h + i4, t, b0, b1);
                        mma_16816(acc[t], A[i4], b0, b1);
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const float c0 = cofs[gi * kNegcStride + 8 * t + 2 * q];
                const float c1 = cofs[gi * kNegcStride + 8 * t + 2 * q + 1];
                yacc[t][0] = fmaf(csa[u], acc[t][0] - c0, yacc[t][0]);
                yacc[t][1] = fmaf(csa[u], acc[t][1] - c1, yacc[t][1]);
                yacc[t][2] = fmaf(csb[u], acc[t][2] - c0, yacc[t][2]);
                yacc[t][3] = fmaf(csb[u], acc[t][3] - c1, yacc[t][3]);
            }
        }
    }

    // 4. Epilogue: reduce over the cluster's K-slices, then write.
    auto emit = [&](int64_t row, int tok, float v) {
        if (row >= a.rows || tok >= M) return;
        if (kResidualPass) {
            a.res_out[int64_t(tok) * a.rows + row] = v;
        } else {
            if (a.res_slot) {
                const int32_t s = a.res_slot[row];
                if (s >= 0 && s < a.r) v += a.res_in[int64_t(tok) * a.r + s];
            }
            a.y[int64_t(tok) * a.rows + row] = __float2half_rn(v);
        }
    };

    if (a.split == 1) {
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            emit(ra, 8 * t + 2 * q, yacc[t][0]);
            emit(ra, 8 * t + 2 * q + 1, yacc[t][1]);
            emit(rb, 8 * t + 2 * q, yacc[t][2]);
            emit(rb, 8 * t + 2 * q + 1, yacc[t][3]);
        }
        return;
    }

    const int lr_a = warp * 16 + rr, lr_b = lr_a + 8;
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        red[lr_a * 16 + 8 * t + 2 * q] = yacc[t][0];
        red[lr_a * 16 + 8 * t + 2 * q + 1] = yacc[t][1];
        red[lr_b * 16 + 8 * t + 2 * q] = yacc[t][2];
        red[lr_b * 16 + 8 * t + 2 * q + 1] = yacc[t][3];
    }
    cluster_sync_all();
    const uint32_t me = cluster_rank();
    const int rows_per_rank = (kRowsPerCta + a.split - 1) / a.split;
    const int lr0 = int(me) * rows_per_rank;
    for (int idx = threadIdx.x; idx < rows_per_rank * M; idx += kThreads) {
        const int lr = lr0 + idx / M, tok = idx % M;
        if (lr >= kRowsPerCta) break;
        float s = 0.f;
        for (int c = 0; c < a.split; ++c) s += ld_dsmem_f32(red + lr * 16 + tok, uint32_t(c));
        emit(block_row0 + lr, tok, s);
    }
    cluster_sync_all();   // keep this CTA's shared memory alive until every rank has read it
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
    int split, gpc, NT;
    size_t smem;
};

Plan plan_for(int64_t rows, int64_t K, int M) {
    Plan p;
    p.NT = M <= 8 ? 1 : 2;
    const int G = int(K / kGroup);
    const int64_t blocks = (rows + kRowsPerCta - 1) / kRowsPerCta;
    const int gpc_smem = std::max(1, kSmemBudget / (M * kGroup * int(sizeof(__half)) + kNegcStride * 4));
    const int min_split = (G + gpc_smem - 1) / gpc_smem;
    const int64_t target = 4LL * sm_count();
    const int par = int(std::min<int64_t>(kMaxSplit, (target + blocks - 1) / blocks));
    int split = std::max(min_split, env_split() > 0 ? env_split() : par);
    split = std::max(1, std::min(split, std::min(kMaxSplit, G)));
    p.gpc = (G + split - 1) / split;
    p.split = (G + p.gpc - 1) / p.gpc;
    p.smem = size_t(M) * p.gpc * kGroup * sizeof(__half) + size_t(p.gpc) * kNegcStride * sizeof(float) +
             size_t(kRowsPerCta) * 16 * sizeof(float);
    return p;
}

template <int NT, bool kRes>
tern_status launch_pass(const GemvArgs& args, const Plan& p, int64_t blocks, cudaStream_t stream) {
    auto kernel = gemv_kernel<NT, kRes>;
    static std::mutex mu;
    static bool configured[64] = {false};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return TERN_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!configured[dev]) {
            if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024) !=
                    cudaSuccess ||
                cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
                return TERN_ERR_CUDA;
            configured[dev] = true;
        }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(p.split), unsigned(blocks), 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = unsigned(p.split);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = p.split > 1 ? 1 : 0;
    GemvArgs a = args;
    a.gpc = p.gpc;
    a.split = p.split;
    if (cudaLaunchKernelEx(&cfg, kernel, a) != cudaSuccess) return TERN_ERR_CUDA;
    return TERN_OK;
}

template <bool kRes>
tern_status run_pass(const GemvArgs& args, cudaStream_t stream) {
    const Plan p = plan_for(args.rows, args.K, args.M);
    if (p.smem > 200 * 1024) return TERN_ERR_SHAPE;
    const int64_t blocks = (args.rows + kRowsPerCta - 1) / kRowsPerCta;
    if (blocks > 65535) return TERN_ERR_SHAPE;
    return p.NT == 1 ? launch_pass<1, kRes>(args, p, blocks, stream) : launch_pass<2, kRes>(args, p, blocks, stream);
}

}  // namespace

size_t gemv_workspace_bytes(const tern_weight& w, int64_t M) {
    if (w.r <= 0 || M <= 0) return 0;
    return size_t(M) * size_t(w.r) * sizeof(float);
}

tern_status gemv_launch(const tern_weight& w, const __half* x, int M, __half* y, float* res_ws, cudaStream_t stream) {
    GemvArgs base = {};
    base.x = x;
    base.K = w.K;
    base.G = int32_t(w.K / kGroup);
    base.M = M;
    if (w.r > 0) {
        GemvArgs ra = base;
        ra.plane = w.plane2;
        ra.scale = reinterpret_cast<const __half*>(w.scale2);
        ra.rows = w.r;
        ra.res_out = res_ws;
        const tern_status st = run_pass<true>(ra, stream);
        if (st != TERN_OK) return st;
    }
    GemvArgs ma = base;
    ma.plane = w.plane1;
    ma.scale = reinterpret_cast<const __half*>(w.scale1);
    ma.rows = w.N;
    ma.y = y;
    if (w.r > 0) {
        ma.res_in = res_ws;
        ma.res_slot = w.res_slot;
        ma.r = w.r;
    }
    return run_pass<false>(ma, stream);
}

}  // namespace tern
