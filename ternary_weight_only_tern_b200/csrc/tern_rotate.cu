// Activation-side rotation: y = x . blockdiag(R_0, ..., R_{G-1}), one 128 x 128 fp16 block per
// 128-wide group of K.
//
// The pages' KOTMS rotation moves the weights into a ternary-friendly basis with structured
// orthogonal matrices, and inference applies the equivalent rotation to the activations before
// the quantized linear operation ("Post-Training Ternarization of Qwen3-4B", arXiv 2609.01962v1,
// section 4.2; the measured path adds that activation-side matrix operation, section 10.1). The
// structure is not given there; this library reads it as block-diagonal with the method's group
// size, so W' = W R and x' = x R give x' W'^T = x W^T for orthogonal R.
//
// One CTA computes 64 tokens x one group (all 128 output columns): it stages the group's block
// (32 KB) and the tokens' 128 activations in shared memory with cp.async (rows padded to 272
// bytes, so the ldmatrix reads of 8 rows hit 32 distinct banks), and each of its 4 warps runs
// 8 k-steps x 16 n-tiles of mma.sync m16n8k16 (fp16 in, fp32 accumulate) for 16 tokens; the
// result is rounded to fp16 once and, for a warp with 16 real tokens, leaves through its own rows of
// the staged tile as 16-byte stores. Everything is read after griddepcontrol.wait; the dependent
// launch is triggered at entry, so the next kernel's weight loads overlap this one.
#include <mutex>

#include "tern_device.cuh"

namespace tern {
namespace {

using namespace dev;

constexpr int kTokTile = 64;
constexpr int kRotThreads = 128;
constexpr int kPitch = kGroup + 8;                                     // halves per staged row
constexpr size_t kRotSmem = size_t(kGroup + kTokTile) * kPitch * 2;  // R block + x tile

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
    // src-size 0 fills the 16 bytes with zeros (tokens past M)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__global__ void __launch_bounds__(kRotThreads) rotate_kernel(const __half* __restrict__ x, int64_t M, int64_t K,
                                                             const __half* __restrict__ R, __half* __restrict__ y) {
    extern __shared__ __align__(16) uint8_t smem_rot[];
    const uint32_t sR = smem_u32(smem_rot);
    const uint32_t sX = sR + kGroup * kPitch * 2;
    const int64_t m0 = int64_t(blockIdx.x) * kTokTile;
    const int64_t g = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    grid_launch_dependents();

    grid_dependency_wait();     // x (and R) may be written by the previous kernel
    // the group's block: 128 rows of 256 bytes, 16 chunks of 16 bytes each
    const __half* Rg = R + g * kGroup * kGroup;
    for (int c = tid; c < kGroup * 16; c += kRotThreads) {
        const int row = c >> 4, col = c & 15;
        cp_async16(sR + (row * kPitch + col * 8) * 2, Rg + row * kGroup + col * 8, true);
    }
    for (int c = tid; c < kTokTile * 16; c += kRotThreads) {
        const int row = c >> 4, col = c & 15;
        const bool valid = m0 + row < M;
        const __half* src = x + (valid ? (m0 + row) * K : 0) + g * kGroup + col * 8;
        cp_async16(sX + (row * kPitch + col * 8) * 2, src, valid);
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
    if (m0 + warp * 16 >= M) return;   // this warp's 16 tokens are all past M

    float acc[16][4];
#pragma unroll
    for (int n = 0; n < 16; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
    // A (16 tokens x 16 k, row-major): lanes 0-15 address rows 0-15 at k0, lanes 16-31 at k0 + 8
    const uint32_t a_base = sX + ((warp * 16 + (lane & 15)) * kPitch + (lane >> 4) * 8) * 2;
    // B (16 k x 16 n from the row-major block, transposed on load): lanes 0-7 rows k0..k0+7 at n0,
    // 8-15 rows k0+8.. at n0, 16-23 rows k0.. at n0 + 8, 24-31 rows k0+8.. at n0 + 8
    const uint32_t b_base = sR + (((lane & 7) + ((lane >> 3) & 1) * 8) * kPitch + (lane >> 4) * 8) * 2;
#pragma unroll
    for (int k = 0; k < kGroup / 16; ++k) {
        uint32_t a[4];
        ldsm_x4(a_base + k * 16 * 2, a);
#pragma unroll
        for (int n = 0; n < 8; ++n) {
            uint32_t b[4];
            ldsm_x4_trans(b_base + (k * 16 * kPitch + n * 16) * 2, b);
            mma_16816(acc[2 * n], a, b[0], b[1]);
            mma_16816(acc[2 * n + 1], a, b[2], b[3]);
        }
    }
    // D: lane holds rows lane/4 and lane/4 + 8 of the warp's tokens, columns 2 (lane % 4) + {0, 1}.
    if (m0 + warp * 16 + 16 > M) {
        // a partial tile (few tokens): each lane stores its pairs
        const int64_t r0 = m0 + warp * 16 + (lane >> 2), r1 = r0 + 8;
        const int c0 = 2 * (lane & 3);
#pragma unroll
        for (int n = 0; n < 16; ++n) {
            const int64_t col = g * kGroup + n * 8 + c0;
            if (r0 < M) *reinterpret_cast<__half2*>(y + r0 * K + col) = __floats2half2_rn(acc[n][0], acc[n][1]);
            if (r1 < M) *reinterpret_cast<__half2*>(y + r1 * K + col) = __floats2half2_rn(acc[n][2], acc[n][3]);
        }
        return;
    }
    // A full tile: the warp's 16 rows go, rounded, into its own rows of the x tile (which only this
    // warp read) and leave as 16-byte stores.
    __syncwarp();
    const uint32_t rowa = sX + ((warp * 16 + (lane >> 2)) * kPitch + 2 * (lane & 3)) * 2;
#pragma unroll
    for (int n = 0; n < 16; ++n) {
        const __half2 v0 = __floats2half2_rn(acc[n][0], acc[n][1]), v1 = __floats2half2_rn(acc[n][2], acc[n][3]);
        asm volatile("st.shared.b32 [%0], %1;" ::"r"(rowa + n * 16), "r"(*reinterpret_cast<const uint32_t*>(&v0))
                     : "memory");
        asm volatile("st.shared.b32 [%0], %1;" ::"r"(rowa + n * 16 + 8 * kPitch * 2),
                     "r"(*reinterpret_cast<const uint32_t*>(&v1))
                     : "memory");
    }
    __syncwarp();
    for (int c = lane; c < 16 * 16; c += 32) {
        const int row = c >> 4, col = c & 15;
        const int64_t m = m0 + warp * 16 + row;
        *reinterpret_cast<uint4*>(y + m * K + g * kGroup + col * 8) =
            lds_u4(sX + ((warp * 16 + row) * kPitch + col * 8) * 2);
    }
}

}  // namespace
}  // namespace tern

using namespace tern;

extern "C" tern_status tern_rotate(const tern_half* x, int64_t M, int64_t K, const tern_half* R, tern_half* y,
                                   tern_stream stream) {
    if (M < 0 || K <= 0 || K % kGroup || K > (int64_t(1) << 20) || M > (int64_t(1) << 31) * kTokTile)
        return TERN_ERR_SHAPE;
    if (M == 0) return TERN_OK;
    if (!x || !R || !y) return TERN_ERR_NULL;
    if (!aligned16(x) || !aligned16(R) || !aligned16(y)) return TERN_ERR_ALIGN;
    const uintptr_t xb = reinterpret_cast<uintptr_t>(x), yb = reinterpret_cast<uintptr_t>(y);
    const size_t bytes = size_t(M) * size_t(K) * 2;
    if (xb < yb + bytes && yb < xb + bytes) return TERN_ERR_SHAPE;   // x and y must not overlap
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned((M + kTokTile - 1) / kTokTile), unsigned(K / kGroup), 1);
    cfg.blockDim = dim3(kRotThreads, 1, 1);
    cfg.dynamicSmemBytes = kRotSmem;
    cfg.stream = as_cuda(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    static std::mutex mu;
    static bool configured[64] = {false};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return TERN_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!configured[dev]) {
            if (cudaFuncSetAttribute(rotate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kRotSmem)) !=
                cudaSuccess)
                return TERN_ERR_CUDA;
            configured[dev] = true;
        }
    }
    if (cudaLaunchKernelEx(&cfg, rotate_kernel, reinterpret_cast<const __half*>(x), M, K,
                           reinterpret_cast<const __half*>(R), reinterpret_cast<__half*>(y)) != cudaSuccess)
        return TERN_ERR_CUDA;
    return TERN_OK;
}
