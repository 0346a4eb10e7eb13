// The ternarization fit: dense fp16 W -> ternary planes, fp16 scales and (optionally) a per-group
// offset, one (row, 128-wide group) at a time.
//
// E2M-ATQ fits an asymmetric offset and two ternary planes with scales, then refines them for 15
// iterations with the ternary supports held fixed ("Post-Training Ternarization of Qwen3-4B",
// arXiv 2609.01962v1, section 4.3); its equations are not given. This library reads it as:
//   mu  = mean of the group (with an offset; else 0), r = w - mu;
//   T1  = sign(r) where |r| > 0.7 mean|r| (the threshold rule of ternary weight networks),
//   a1  = mean of |r| over T1's support;
//   T2, a2 the same on e = r - a1 T1, for rows that carry a second plane;
//   then `iters` rounds of: mu, a1, a2 each set to its least-squares value with the others and
//   both planes fixed.
// Every sum runs over the group's 128 entries in index order in float64, and every operation is
// rounded on its own (the _rn intrinsics are never contracted into a fused multiply-add), so the
// float64 restatement in the tests reaches the same thresholds, planes and scales bit for bit.
//
// One thread per group; a block of 128 threads takes 128 consecutive groups, which are 32 KB of
// contiguous W, staged in shared memory with 16-byte loads (rows padded to 272 bytes). The planes
// are kept as bit masks (support and sign, 4 words each). Offline work, bound by the float64
// dependency chains of the sums.
#include "tern_internal.cuh"

namespace tern {
namespace {

constexpr int kFitThreads = 128;
constexpr int kRowPitch = kGroup * 2 + 16;     // bytes per staged group
constexpr double kTwnRatio = 0.7;

struct Plane {
    uint32_t nz[4], neg[4];   // trit k: support bit k % 32 of nz[k / 32], sign in neg
    __device__ __forceinline__ double t(int k) const {
        const uint32_t b = 1u << (k & 31);
        return (nz[k >> 5] & b) ? ((neg[k >> 5] & b) ? -1.0 : 1.0) : 0.0;
    }
};

__device__ __forceinline__ double wk(const __half* w, int k) { return double(__half2float(w[k])); }

// sign plane of r (given by rk(k)) at 0.7 mean |r|, its support size and mean magnitude on it
template <typename R>
__device__ __forceinline__ void threshold_plane(R rk, Plane& p, int& n, double& a) {
    double abs_sum = 0.0;
    for (int k = 0; k < kGroup; ++k) abs_sum = __dadd_rn(abs_sum, fabs(rk(k)));
    const double delta = __dmul_rn(kTwnRatio, __ddiv_rn(abs_sum, double(kGroup)));
    double s = 0.0;
    n = 0;
    for (int i = 0; i < 4; ++i) p.nz[i] = p.neg[i] = 0u;
    for (int k = 0; k < kGroup; ++k) {
        const double r = rk(k);
        const bool pos = r > delta, negv = r < -delta;
        if (pos || negv) {
            p.nz[k >> 5] |= 1u << (k & 31);
            if (negv) p.neg[k >> 5] |= 1u << (k & 31);
            ++n;
        }
        s = __dadd_rn(s, (pos || negv) ? fabs(r) : 0.0);
    }
    a = n > 0 ? __ddiv_rn(s, double(n)) : 0.0;
}

__global__ void __launch_bounds__(kFitThreads) fit_kernel(const __half* __restrict__ W, int64_t N, int64_t K,
                                                          const int32_t* __restrict__ res_slot, int64_t r,
                                                          int offset, int iters, int8_t* __restrict__ T1,
                                                          __half* __restrict__ s1, __half* __restrict__ mu_out,
                                                          int8_t* __restrict__ T2, __half* __restrict__ s2) {
    __shared__ __align__(16) uint8_t stage[kFitThreads * kRowPitch];
    const int64_t G = K / kGroup, groups = N * G;
    const int64_t first = int64_t(blockIdx.x) * kFitThreads;
    // the block's groups are contiguous in W: 16-byte chunks, 16 per group
    for (int c = threadIdx.x; c < kFitThreads * 16; c += kFitThreads) {
        const int64_t gi = first + (c >> 4);
        if (gi < groups)
            *reinterpret_cast<uint4*>(stage + (c >> 4) * kRowPitch + (c & 15) * 16) =
                __ldg(reinterpret_cast<const uint4*>(W + gi * kGroup) + (c & 15));
    }
    __syncthreads();
    const int64_t gi = first + threadIdx.x;
    if (gi >= groups) return;
    const int64_t n = gi / G, g = gi - n * G;
    const __half* w = reinterpret_cast<const __half*>(stage + threadIdx.x * kRowPitch);
    int slot = -1;
    if (res_slot) {
        const int32_t s = res_slot[n];
        if (s >= 0 && s < r) slot = s;
    }

    double mu = 0.0;
    if (offset) {
        double acc = 0.0;
        for (int k = 0; k < kGroup; ++k) acc = __dadd_rn(acc, wk(w, k));
        mu = __ddiv_rn(acc, double(kGroup));
    }
    Plane p1, p2;
    int n1 = 0, n2 = 0;
    double a1 = 0.0, a2 = 0.0;
    threshold_plane([&](int k) { return __dsub_rn(wk(w, k), mu); }, p1, n1, a1);
    if (slot >= 0) {
        threshold_plane([&](int k) { return __dsub_rn(__dsub_rn(wk(w, k), mu), __dmul_rn(a1, p1.t(k))); }, p2, n2,
                        a2);
    } else {
        for (int i = 0; i < 4; ++i) p2.nz[i] = p2.neg[i] = 0u;
    }
    for (int it = 0; it < iters; ++it) {
        if (offset) {
            double acc = 0.0;
            for (int k = 0; k < kGroup; ++k)
                acc = __dadd_rn(acc, __dsub_rn(__dsub_rn(wk(w, k), __dmul_rn(a1, p1.t(k))), __dmul_rn(a2, p2.t(k))));
            mu = __ddiv_rn(acc, double(kGroup));
        }
        double acc = 0.0;
        for (int k = 0; k < kGroup; ++k)
            acc = __dadd_rn(acc, __dmul_rn(__dsub_rn(__dsub_rn(wk(w, k), mu), __dmul_rn(a2, p2.t(k))), p1.t(k)));
        a1 = n1 > 0 ? __ddiv_rn(acc, double(n1)) : 0.0;
        acc = 0.0;
        for (int k = 0; k < kGroup; ++k)
            acc = __dadd_rn(acc, __dmul_rn(__dsub_rn(__dsub_rn(wk(w, k), mu), __dmul_rn(a1, p1.t(k))), p2.t(k)));
        a2 = n2 > 0 ? __ddiv_rn(acc, double(n2)) : 0.0;
    }

    // outputs: the trits as int8 (16-byte stores), the scales and offset rounded once to fp16
    int8_t* t1 = T1 + n * K + g * kGroup;
    for (int c = 0; c < kGroup / 16; ++c) {
        uint32_t q[4];
        for (int j = 0; j < 4; ++j) {
            uint32_t v = 0;
            for (int b = 0; b < 4; ++b) {
                const int k = c * 16 + j * 4 + b;
                v |= uint32_t(uint8_t(int8_t(p1.t(k)))) << (8 * b);
            }
            q[j] = v;
        }
        reinterpret_cast<uint4*>(t1)[c] = make_uint4(q[0], q[1], q[2], q[3]);
    }
    s1[n * G + g] = __double2half(a1);
    if (offset) mu_out[n * G + g] = __double2half(mu);
    if (slot >= 0) {
        int8_t* t2 = T2 + int64_t(slot) * K + g * kGroup;
        for (int c = 0; c < kGroup / 16; ++c) {
            uint32_t q[4];
            for (int j = 0; j < 4; ++j) {
                uint32_t v = 0;
                for (int b = 0; b < 4; ++b) {
                    const int k = c * 16 + j * 4 + b;
                    v |= uint32_t(uint8_t(int8_t(p2.t(k)))) << (8 * b);
                }
                q[j] = v;
            }
            reinterpret_cast<uint4*>(t2)[c] = make_uint4(q[0], q[1], q[2], q[3]);
        }
        s2[int64_t(slot) * G + g] = __double2half(a2);
    }
}

}  // namespace
}  // namespace tern

using namespace tern;

extern "C" tern_status tern_fit(const tern_half* W, int64_t N, int64_t K, const int32_t* res_slot, int64_t r,
                                int32_t offset, int32_t iters, int8_t* T1, tern_half* s1, tern_half* mu, int8_t* T2,
                                tern_half* s2, tern_stream stream) {
    if (N < 0 || K <= 0 || K % kGroup || K > (int64_t(1) << 20) || N > (int64_t(1) << 30) || r < 0 || r > N ||
        iters < 0 || iters > 1000)
        return TERN_ERR_SHAPE;
    if (N == 0) return TERN_OK;
    if (!W || !T1 || !s1 || (offset && !mu) || (r > 0 && (!res_slot || !T2 || !s2))) return TERN_ERR_NULL;
    if (!aligned16(W) || !aligned16(T1) || (r > 0 && !aligned16(T2))) return TERN_ERR_ALIGN;
    const int64_t groups = N * (K / kGroup);
    const int64_t blocks = (groups + kFitThreads - 1) / kFitThreads;
    if (blocks > 0x7fffffff) return TERN_ERR_SHAPE;
    fit_kernel<<<unsigned(blocks), kFitThreads, 0, as_cuda(stream)>>>(
        reinterpret_cast<const __half*>(W), N, K, r > 0 ? res_slot : nullptr, r, offset ? 1 : 0, iters, T1,
        reinterpret_cast<__half*>(s1), reinterpret_cast<__half*>(mu), T2, reinterpret_cast<__half*>(s2));
    return cudaGetLastError() == cudaSuccess ? TERN_OK : TERN_ERR_CUDA;
}
