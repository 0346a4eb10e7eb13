// The element-level second plane: packing into its listed form, unpacking, and checks.
//
// The pages give a second ternary plane to the weights of the two most salient of four
// disjoint element masks (the Qwen3-8B scale-up paper, representation paragraph;
// "Post-Training Ternarization of Qwen3-4B", arXiv 2609.01962v1, section 4.4: 3.6 % of a
// recorded projection). The plane T2e [N, K] is zero outside the masks, so it is kept as the
// list of its nonzero trits, one byte each, (k % 128) << 1 | (t < 0), ordered by group, row,
// k. ecount [G, N] holds the number listed per (group, row) and ebase [G * NB + 1]
// (NB = ceil(N / 64)) the index of the first one of each (group, 64-row block), so a block of
// 64 rows finds its trits of one group as one contiguous run. The layout is this library's own.
//
// One CTA of 64 threads per (64-row block, group), one thread per row: it reads the row's 128
// trits of the group (eight 16-byte loads) and writes or reads its run. Offline work,
// memory-bound; the block bases are an exclusive scan over G * NB block totals done on the host
// between the count and the fill kernels.
#include <vector>

#include "tern_internal.cuh"

namespace tern {
namespace {

constexpr int kEBlock = kElemBlock;
constexpr unsigned kBadTrit = 1u;
constexpr unsigned kBadMeta = 4u;

// inclusive sum of v over the 64 threads of the block in thread order, and the block total
__device__ __forceinline__ int block64_scan(int v, int* total) {
    __shared__ int warp_total[2];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
    }
    if (lane == 31) warp_total[warp] = incl;
    __syncthreads();
    *total = warp_total[0] + warp_total[1];
    return incl + (warp ? warp_total[0] : 0);
}

__global__ void __launch_bounds__(kEBlock) elem_count_kernel(const int8_t* __restrict__ t, int64_t N, int64_t K,
                                                             uint8_t* __restrict__ ecount,
                                                             int32_t* __restrict__ block_total,
                                                             unsigned int* status) {
    const int64_t b = blockIdx.x, g = blockIdx.y;
    const int64_t n = b * kEBlock + threadIdx.x;
    int c = 0;
    bool bad = false;
    if (n < N) {
        const int4* src = reinterpret_cast<const int4*>(t + n * K + g * kGroup);
#pragma unroll
        for (int i = 0; i < kGroup / 16; ++i) {
            const int4 v = __ldg(src + i);
            const int8_t* p = reinterpret_cast<const int8_t*>(&v);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const bool ok = p[j] >= -1 && p[j] <= 1;
                bad |= !ok;
                c += (ok && p[j] != 0) ? 1 : 0;
            }
        }
        ecount[g * N + n] = static_cast<uint8_t>(c);
    }
    int total = 0;
    block64_scan(c, &total);
    if (threadIdx.x == 0) block_total[g * gridDim.x + b] = total;
    if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(status, kBadTrit);
}

__global__ void __launch_bounds__(kEBlock) elem_fill_kernel(const int8_t* __restrict__ t, int64_t N, int64_t K,
                                                            const uint8_t* __restrict__ ecount,
                                                            const int32_t* __restrict__ ebase,
                                                            uint8_t* __restrict__ eidx) {
    const int64_t b = blockIdx.x, g = blockIdx.y;
    const int64_t n = b * kEBlock + threadIdx.x;
    const int c = n < N ? ecount[g * N + n] : 0;
    int total = 0;
    const int excl = block64_scan(c, &total) - c;
    if (n >= N) return;
    int64_t pos = int64_t(ebase[g * gridDim.x + b]) + excl;
    const int8_t* src = t + n * K + g * kGroup;
    for (int k = 0; k < kGroup; ++k) {
        const int8_t v = src[k];
        if (v == 1 || v == -1) eidx[pos++] = static_cast<uint8_t>((k << 1) | (v < 0 ? 1 : 0));
    }
}

// Reads the listed form back (out may be null: checks only). Trits at indices outside
// [0, nnz2) are skipped; every inconsistency sets kBadMeta.
__global__ void __launch_bounds__(kEBlock) elem_unpack_kernel(const uint8_t* __restrict__ ecount,
                                                              const int32_t* __restrict__ ebase,
                                                              const uint8_t* __restrict__ eidx, int64_t nnz2,
                                                              int64_t N, int64_t K, int8_t* __restrict__ out,
                                                              unsigned int* status) {
    const int64_t b = blockIdx.x, g = blockIdx.y;
    const int64_t n = b * kEBlock + threadIdx.x;
    const int64_t cell = g * gridDim.x + b;
    const int c = n < N ? ecount[g * N + n] : 0;
    int total = 0;
    const int excl = block64_scan(c, &total) - c;
    const int64_t base = ebase[cell], next = ebase[cell + 1];
    bool bad = c > kGroup;
    if (threadIdx.x == 0) {
        bad |= (next - base) != total;
        if (cell == 0) bad |= base != 0;
        if (cell + 1 == int64_t(gridDim.x) * gridDim.y) bad |= next != nnz2;
    }
    if (n < N) {
        int8_t* dst = out ? out + n * K + g * kGroup : nullptr;
        if (dst)
            for (int i = 0; i < kGroup / 16; ++i) reinterpret_cast<int4*>(dst)[i] = make_int4(0, 0, 0, 0);
        int last = -1;
        for (int e = 0; e < c; ++e) {
            const int64_t i = base + excl + e;
            if (i < 0 || i >= nnz2) {
                bad = true;
                continue;
            }
            const int v = eidx[i], k = v >> 1;
            bad |= k <= last;
            last = k;
            if (dst) dst[k] = (v & 1) ? int8_t(-1) : int8_t(1);
        }
    }
    if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(status, kBadMeta);
}

tern_status read_status(unsigned int* slot, cudaStream_t st, unsigned int* v) {
    if (cudaGetLastError() != cudaSuccess) return TERN_ERR_CUDA;
    return read_flag_slot(slot, st, v);
}

bool elem_shape_ok(int64_t N, int64_t K) {
    return N >= 0 && K > 0 && K % kGroup == 0 && K <= (int64_t(1) << 20) && N <= (int64_t(1) << 26) &&
           K / kGroup <= 65535 && (N + kEBlock - 1) / kEBlock <= 0x7fffffff;
}

}  // namespace

tern_status elem_check(const tern_weight& w, cudaStream_t st) {
    const int64_t G = w.K / kGroup, NB = (w.N + kEBlock - 1) / kEBlock;
    if (w.N == 0) return TERN_OK;
    unsigned int* slot = acquire_flag_slot(st);
    if (!slot) return TERN_ERR_CUDA;
    elem_unpack_kernel<<<dim3(unsigned(NB), unsigned(G)), kEBlock, 0, st>>>(w.ecount, w.ebase, w.eidx, w.nnz2, w.N,
                                                                         w.K, nullptr, slot);
    unsigned int v = 0;
    const tern_status s = read_status(slot, st, &v);
    if (s != TERN_OK) return s;
    return v ? TERN_ERR_ELEM : TERN_OK;
}

}  // namespace tern

using namespace tern;

extern "C" tern_status tern_pack_elem(const int8_t* t, int64_t N, int64_t K, uint8_t* ecount, int32_t* ebase,
                                      uint8_t* eidx, int64_t eidx_bytes, int64_t* nnz2, tern_stream s) {
    if (!nnz2) return TERN_ERR_NULL;
    *nnz2 = 0;
    if (!elem_shape_ok(N, K)) return TERN_ERR_SHAPE;
    if (!ebase) return TERN_ERR_NULL;
    if (!aligned16(ebase)) return TERN_ERR_ALIGN;
    cudaStream_t st = as_cuda(s);
    const int64_t G = K / kGroup, NB = (N + kEBlock - 1) / kEBlock, cells = G * NB;
    if (N == 0) {
        if (cudaMemsetAsync(ebase, 0, sizeof(int32_t), st) != cudaSuccess) return TERN_ERR_CUDA;
        return cudaStreamSynchronize(st) == cudaSuccess ? TERN_OK : TERN_ERR_CUDA;
    }
    if (!t || !ecount) return TERN_ERR_NULL;
    if (!aligned16(t) || !aligned16(ecount) || (eidx && !aligned16(eidx))) return TERN_ERR_ALIGN;

    unsigned int* slot = acquire_flag_slot(st);
    if (!slot) return TERN_ERR_CUDA;
    const dim3 grid{unsigned(NB), unsigned(G), 1u};
    elem_count_kernel<<<grid, kEBlock, 0, st>>>(t, N, K, ecount, ebase, slot);
    unsigned int v = 0;
    tern_status rs = read_status(slot, st, &v);
    if (rs != TERN_OK) return rs;
    // exclusive scan of the block totals, on the host
    std::vector<int32_t> base(size_t(cells) + 1);
    if (cudaMemcpyAsync(base.data(), ebase, size_t(cells) * sizeof(int32_t), cudaMemcpyDeviceToHost, st) !=
            cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return TERN_ERR_CUDA;
    int64_t run = 0;
    for (int64_t i = 0; i < cells; ++i) {
        const int64_t c = base[size_t(i)];
        base[size_t(i)] = int32_t(run);
        run += c;
        if (run > 0x7fffffff) return TERN_ERR_SHAPE;
    }
    base[size_t(cells)] = int32_t(run);
    if (cudaMemcpyAsync(ebase, base.data(), size_t(cells + 1) * sizeof(int32_t), cudaMemcpyHostToDevice, st) !=
            cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return TERN_ERR_CUDA;
    *nnz2 = run;
    const tern_status trit_status = v ? TERN_ERR_BAD_TRIT : TERN_OK;
    if (!eidx) return trit_status;
    const int64_t padded = (run + 15) / 16 * 16;
    if (eidx_bytes < padded) return TERN_ERR_WORKSPACE;
    if (padded > run && cudaMemsetAsync(eidx + run, 0, size_t(padded - run), st) != cudaSuccess) return TERN_ERR_CUDA;
    elem_fill_kernel<<<grid, kEBlock, 0, st>>>(t, N, K, ecount, ebase, eidx);
    if (cudaGetLastError() != cudaSuccess || cudaStreamSynchronize(st) != cudaSuccess) return TERN_ERR_CUDA;
    return trit_status;
}

extern "C" tern_status tern_unpack_elem(const uint8_t* ecount, const int32_t* ebase, const uint8_t* eidx,
                                        int64_t nnz2, int64_t N, int64_t K, int8_t* out, tern_stream s) {
    if (!elem_shape_ok(N, K) || nnz2 < 0 || nnz2 > 0x7fffffff) return TERN_ERR_SHAPE;
    if (N == 0) return TERN_OK;
    if (!ecount || !ebase || !out || (nnz2 > 0 && !eidx)) return TERN_ERR_NULL;
    if (!aligned16(ecount) || !aligned16(ebase) || !aligned16(out) || (eidx && !aligned16(eidx)))
        return TERN_ERR_ALIGN;
    cudaStream_t st = as_cuda(s);
    const int64_t G = K / kGroup, NB = (N + kEBlock - 1) / kEBlock;
    unsigned int* slot = acquire_flag_slot(st);
    if (!slot) return TERN_ERR_CUDA;
    elem_unpack_kernel<<<dim3(unsigned(NB), unsigned(G)), kEBlock, 0, st>>>(ecount, ebase, eidx, nnz2, N, K, out,
                                                                         slot);
    unsigned int v = 0;
    const tern_status rs = read_status(slot, st, &v);
    if (rs != TERN_OK) return rs;
    return v ? TERN_ERR_ELEM : TERN_OK;
}
