// Packing of ternary planes: int8 trits <-> 2-bit execution codes and base-3 storage bytes,
// and the device-side check of a weight descriptor.
//
// The packed format persists the discrete planes (not a floating reconstruction); that is
// what makes the pages' packing lossless ("Post-Training Ternarization of Qwen3-4B",
// arXiv 2609.01962v1, section 9.1 and Table 6; section 9.2 shows what is lost when a plane
// is dropped). The two byte layouts are this library's own:
//   exec : code c = t + 1, 16 codes per uint32, trit k at bits 2*(k % 16), row-major.
//   store: byte = sum_{i<5} (t_i + 1) * 3^i, ceil(K/5) bytes per row, padding digit 1.
//
// Every kernel is elementwise and memory-bound; these calls are offline (conversion time).
// Invalid input is reported through a device status word (no trap), and the call returns
// after the stream drains.
#include <atomic>
#include <mutex>

#include "tern_device.cuh"

namespace tern {

// ------------------------------------------------------------------ status words
// A small ring of device words; each synchronous call takes its own slot so that calls
// on different streams or host threads do not share one.
constexpr int kFlagSlots = 256;
__device__ unsigned int g_status_words[kFlagSlots];
__device__ unsigned int g_async_status;            // set by tern_linear kernels whose bounded wait ran out

namespace {
std::atomic<unsigned int> g_next_slot{0};
std::mutex g_addr_mu;
unsigned int* g_slot_base[64] = {nullptr};
}  // namespace

unsigned int* async_status_word() {
    static unsigned int* addr[64] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(g_addr_mu);
    if (!addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_async_status) != cudaSuccess) return nullptr;
        addr[dev] = static_cast<unsigned int*>(p);
    }
    return addr[dev];
}

unsigned int* acquire_flag_slot(cudaStream_t stream) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    unsigned int* base = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_addr_mu);
        if (!g_slot_base[dev]) {
            void* p = nullptr;
            if (cudaGetSymbolAddress(&p, g_status_words) != cudaSuccess) return nullptr;
            g_slot_base[dev] = static_cast<unsigned int*>(p);
        }
        base = g_slot_base[dev];
    }
    unsigned int* slot = base + (g_next_slot.fetch_add(1) % kFlagSlots);
    if (cudaMemsetAsync(slot, 0, sizeof(unsigned int), stream) != cudaSuccess) return nullptr;
    return slot;
}

tern_status read_flag_slot(unsigned int* slot, cudaStream_t stream, unsigned int* value) {
    unsigned int h = 0;
    if (cudaMemcpyAsync(&h, slot, sizeof(h), cudaMemcpyDeviceToHost, stream) != cudaSuccess) return TERN_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return TERN_ERR_CUDA;
    *value = h;
    return TERN_OK;
}

namespace {

constexpr unsigned kBadInput = 1u;
constexpr unsigned kBadResidual = 2u;

__device__ __forceinline__ uint32_t trit_code(int8_t t, bool& bad) {
    // c = t + 1; anything outside {-1, 0, +1} becomes the code of 0 and is reported
    const bool ok = (t >= -1) && (t <= 1);
    bad |= !ok;
    return ok ? static_cast<uint32_t>(t + 1) : 1u;
}

// One thread per output word: 16 int8 trits (one 16-byte load) -> one uint32.
__global__ void pack_exec_kernel(const int8_t* __restrict__ t, int64_t n_words, uint32_t* __restrict__ out,
                                 unsigned int* status) {
    bool bad = false;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n_words;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int4 v = __ldg(reinterpret_cast<const int4*>(t) + i);
        const int8_t* b = reinterpret_cast<const int8_t*>(&v);
        uint32_t w = 0;
#pragma unroll
        for (int k = 0; k < 16; ++k) w |= trit_code(b[k], bad) << (2 * k);
        out[i] = w;
    }
    if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(status, kBadInput);
}

// One thread per word: uint32 -> 16 int8 trits (one 16-byte store). Code 3 -> 0, reported.
__global__ void unpack_exec_kernel(const uint32_t* __restrict__ p, int64_t n_words, int8_t* __restrict__ out,
                                   unsigned int* status) {
    bool bad = false;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n_words;
         i += (int64_t)gridDim.x * blockDim.x) {
        const uint32_t w = __ldg(p + i);
        int4 v;
        int8_t* b = reinterpret_cast<int8_t*>(&v);
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const uint32_t c = (w >> (2 * k)) & 3u;
            bad |= (c == 3u);
            b[k] = (c == 3u) ? int8_t(0) : static_cast<int8_t>(static_cast<int>(c) - 1);
        }
        reinterpret_cast<int4*>(out)[i] = v;
    }
    if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(status, kBadInput);
}

// One thread per output byte (row, j): trits 5j .. 5j+4 of the row, padding past K = digit 1.
__global__ void pack_store_kernel(const int8_t* __restrict__ t, int64_t rows, int64_t K, int64_t bytes_per_row,
                                  uint8_t* __restrict__ out, unsigned int* status) {
    bool bad = false;
    const int64_t total = rows * bytes_per_row;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t row = i / bytes_per_row;
        const int64_t j = i - row * bytes_per_row;
        const int8_t* src = t + row * K + 5 * j;
        uint32_t v = 0, pow3 = 1;
#pragma unroll
        for (int d = 0; d < kTritsPerByte; ++d) {
            const uint32_t digit = (5 * j + d < K) ? trit_code(src[d], bad) : 1u;
            v += digit * pow3;
            pow3 *= 3u;
        }
        out[i] = static_cast<uint8_t>(v);
    }
    if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(status, kBadInput);
}

// One thread per byte: base-3 digits, least significant first. Bytes >= 243 decode as five 0
// trits; a padding digit (position >= K) other than 1 is non-canonical. Both are reported.
__global__ void unpack_store_kernel(const uint8_t* __restrict__ b, int64_t rows, int64_t K, int64_t bytes_per_row,
                                    int8_t* __restrict__ out, unsigned int* status) {
    bool bad = false;
    const int64_t total = rows * bytes_per_row;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t row = i / bytes_per_row;
        const int64_t j = i - row * bytes_per_row;
        uint32_t v = b[i];
        const bool bad_byte = v >= 243u;
        bad |= bad_byte;
        int8_t* dst = out + row * K + 5 * j;
#pragma unroll
        for (int d = 0; d < kTritsPerByte; ++d) {
            const uint32_t digit = bad_byte ? 1u : (v % 3u);
            v /= 3u;
            if (5 * j + d < K) dst[d] = static_cast<int8_t>(static_cast<int>(digit) - 1);
            else bad |= (digit != 1u);
        }
    }
    if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(status, kBadInput);
}

// Checks of a descriptor's device data (see tern_weight_validate).
__global__ void validate_codes_kernel(const uint32_t* __restrict__ p, int64_t n_words, unsigned int* status) {
    bool bad = false;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n_words;
         i += (int64_t)gridDim.x * blockDim.x) {
        const uint32_t w = __ldg(p + i);
        // a code is 3 exactly when both of its bits are set
        bad |= ((w & (w >> 1) & 0x55555555u) != 0u);
    }
    if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(status, kBadInput);
}

__global__ void validate_residual_kernel(const int32_t* __restrict__ rows, const int32_t* __restrict__ slot,
                                         int64_t N, int64_t r, unsigned int* status) {
    bool bad = false;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < N + r;
         i += (int64_t)gridDim.x * blockDim.x) {
        if (i < N) {
            const int32_t s = slot[i];
            if (s < -1 || s >= r) bad = true;
            else if (s >= 0 && rows[s] != i) bad = true;
        } else {
            const int64_t k = i - N;
            const int32_t n = rows[k];
            if (n < 0 || n >= N) bad = true;
            else if (slot[n] != k) bad = true;
            if (k + 1 < r && rows[k + 1] <= n) bad = true;
        }
    }
    if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(status, kBadResidual);
}

// Residual-row metadata: the sorted rows R -> the slot map (execution form) and the row bitmap
// (storage form), and back.
__global__ void slot_fill_kernel(int32_t* __restrict__ slot, int64_t N) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < N; i += (int64_t)gridDim.x * blockDim.x)
        slot[i] = -1;
}

__global__ void slot_scatter_kernel(const int32_t* __restrict__ rows, int64_t r, int64_t N, int32_t* __restrict__ slot,
                                    unsigned int* status) {
    bool bad = false;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < r; i += (int64_t)gridDim.x * blockDim.x) {
        const int32_t n = rows[i];
        if (n < 0 || n >= N) {
            bad = true;
            continue;
        }
        if (i + 1 < r && rows[i + 1] <= n) bad = true;   // not strictly increasing
        slot[n] = int32_t(i);
    }
    if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(status, kBadResidual);
}

// Byte j of the bitmap: bit b is set when row 8 j + b has a slot.
__global__ void bitmap_from_slots_kernel(const int32_t* __restrict__ slot, int64_t N, uint8_t* __restrict__ bitmap) {
    const int64_t nbytes = (N + 7) / 8;
    for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < nbytes;
         j += (int64_t)gridDim.x * blockDim.x) {
        uint32_t v = 0;
        for (int b = 0; b < 8; ++b) {
            const int64_t n = 8 * j + b;
            if (n < N && slot[n] >= 0) v |= 1u << b;
        }
        bitmap[j] = uint8_t(v);
    }
}

// One CTA walks the bitmap in order, kRowsThreads bytes per round: each thread counts its
// byte's rows, a block scan gives each its first index, and the rows (and slots) are written.
// count receives r; a bit set past row N - 1 is reported as non-canonical.
constexpr int kRowsThreads = 1024;
__global__ void __launch_bounds__(kRowsThreads) rows_from_bitmap_kernel(const uint8_t* __restrict__ bitmap, int64_t N,
                                                                        int32_t* __restrict__ rows, int64_t r_cap,
                                                                        int32_t* __restrict__ slot,
                                                                        unsigned int* count, unsigned int* status) {
    __shared__ unsigned int warp_tot[kRowsThreads / 32];
    __shared__ unsigned int base_s;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t nbytes = (N + 7) / 8;
    if (threadIdx.x == 0) base_s = 0;
    __syncthreads();
    bool bad = false;
    for (int64_t j0 = 0; j0 < nbytes; j0 += kRowsThreads) {
        const int64_t j = j0 + threadIdx.x;
        uint32_t v = j < nbytes ? bitmap[j] : 0u;
        const int valid = int(min(int64_t(8), N - 8 * j));   // rows held by this byte
        if (j < nbytes && valid < 8) {
            bad |= (v >> valid) != 0u;
            v &= (1u << valid) - 1u;
        }
        const unsigned int c = __popc(v);
        unsigned int inc = c;   // inclusive scan within the warp
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned int u = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += u;
        }
        if (lane == 31) warp_tot[warp] = inc;
        __syncthreads();
        if (warp == 0) {
            unsigned int t = warp_tot[lane], ti = t;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned int u = __shfl_up_sync(0xffffffffu, ti, o);
                if (lane >= o) ti += u;
            }
            warp_tot[lane] = ti - t;   // exclusive prefix of the warps
        }
        __syncthreads();
        unsigned int idx = base_s + warp_tot[warp] + inc - c;
        if (j < nbytes) {
            for (int b = 0; b < valid; ++b) {
                const int64_t n = 8 * j + b;
                const bool set = (v >> b) & 1u;
                if (set && rows && int64_t(idx) < r_cap) rows[idx] = int32_t(n);
                if (slot) slot[n] = set ? int32_t(idx) : -1;
                idx += set ? 1u : 0u;
            }
        }
        __syncthreads();
        if (threadIdx.x == kRowsThreads - 1) base_s += warp_tot[warp] + inc;
        __syncthreads();
    }
    if (threadIdx.x == 0) *count = base_s;
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(status, kBadInput);
}

// The failure path of the bounded waits, on its own: one thread waits on a barrier that nothing
// completes and, when the bound runs out, records the timeout as a linear kernel would.
__global__ void selftest_timeout_kernel(uint64_t cycles, unsigned int* status) {
    __shared__ uint64_t bar;
    dev::mbar_init(&bar, 1);
    dev::fence_barrier_init();
    if (!dev::mbar_wait_for(&bar, 0, cycles) && status) atomicOr(status, 1u);
}

int grid_for(int64_t items, int threads) {
    const int64_t want = (items + threads - 1) / threads;
    const int64_t cap = static_cast<int64_t>(sm_count()) * 32;
    return static_cast<int>(want < 1 ? 1 : (want > cap ? cap : want));
}

template <typename Launch>
tern_status run_checked(cudaStream_t stream, Launch&& launch, tern_status on_flag) {
    unsigned int* slot = acquire_flag_slot(stream);
    if (!slot) return TERN_ERR_CUDA;
    launch(slot);
    if (cudaGetLastError() != cudaSuccess) return TERN_ERR_CUDA;
    unsigned int v = 0;
    const tern_status st = read_flag_slot(slot, stream, &v);
    if (st != TERN_OK) return st;
    if (v & kBadResidual) return TERN_ERR_RESIDUAL;
    return v ? on_flag : TERN_OK;
}

}  // namespace
}  // namespace tern

using namespace tern;

extern "C" tern_status tern_pack_exec(const int8_t* t, int64_t rows, int64_t K, uint32_t* out, tern_stream s) {
    if (rows < 0 || K < 0 || K % kCodesPerWord) return TERN_ERR_SHAPE;
    if (rows == 0 || K == 0) return TERN_OK;
    if (!t || !out) return TERN_ERR_NULL;
    if (!aligned16(t) || !aligned16(out)) return TERN_ERR_ALIGN;
    const int64_t n = rows * (K / kCodesPerWord);
    cudaStream_t st = as_cuda(s);
    return run_checked(st, [&](unsigned int* f) {
        pack_exec_kernel<<<grid_for(n, 256), 256, 0, st>>>(t, n, out, f);
    }, TERN_ERR_BAD_TRIT);
}

extern "C" tern_status tern_unpack_exec(const uint32_t* p, int64_t rows, int64_t K, int8_t* out, tern_stream s) {
    if (rows < 0 || K < 0 || K % kCodesPerWord) return TERN_ERR_SHAPE;
    if (rows == 0 || K == 0) return TERN_OK;
    if (!p || !out) return TERN_ERR_NULL;
    if (!aligned16(p) || !aligned16(out)) return TERN_ERR_ALIGN;
    const int64_t n = rows * (K / kCodesPerWord);
    cudaStream_t st = as_cuda(s);
    return run_checked(st, [&](unsigned int* f) {
        unpack_exec_kernel<<<grid_for(n, 256), 256, 0, st>>>(p, n, out, f);
    }, TERN_ERR_BAD_CODE);
}

extern "C" tern_status tern_pack_store(const int8_t* t, int64_t rows, int64_t K, uint8_t* out, tern_stream s) {
    if (rows < 0 || K < 0) return TERN_ERR_SHAPE;
    if (rows == 0 || K == 0) return TERN_OK;
    if (!t || !out) return TERN_ERR_NULL;
    const int64_t bpr = (K + kTritsPerByte - 1) / kTritsPerByte;
    cudaStream_t st = as_cuda(s);
    return run_checked(st, [&](unsigned int* f) {
        pack_store_kernel<<<grid_for(rows * bpr, 256), 256, 0, st>>>(t, rows, K, bpr, out, f);
    }, TERN_ERR_BAD_TRIT);
}

extern "C" tern_status tern_unpack_store(const uint8_t* b, int64_t rows, int64_t K, int8_t* out, tern_stream s) {
    if (rows < 0 || K < 0) return TERN_ERR_SHAPE;
    if (rows == 0 || K == 0) return TERN_OK;
    if (!b || !out) return TERN_ERR_NULL;
    const int64_t bpr = (K + kTritsPerByte - 1) / kTritsPerByte;
    cudaStream_t st = as_cuda(s);
    return run_checked(st, [&](unsigned int* f) {
        unpack_store_kernel<<<grid_for(rows * bpr, 256), 256, 0, st>>>(b, rows, K, bpr, out, f);
    }, TERN_ERR_BAD_CODE);
}

extern "C" tern_status tern_weight_validate(const tern_weight* w, tern_stream s) {
    if (!w) return TERN_ERR_NULL;
    if (w->N < 0 || w->K <= 0 || w->K % kGroup || w->group != kGroup || w->r < 0 || w->r > w->N)
        return TERN_ERR_SHAPE;
    if (w->N == 0) return TERN_OK;
    if (!w->plane1 || !w->scale1) return TERN_ERR_NULL;
    if (w->r > 0 && (!w->plane2 || !w->scale2 || !w->res_rows || !w->res_slot)) return TERN_ERR_NULL;
    cudaStream_t st = as_cuda(s);
    const int64_t n1 = w->N * (w->K / kCodesPerWord);
    const int64_t n2 = w->r * (w->K / kCodesPerWord);
    if (w->ecount && (w->r > 0 || !w->ebase || !w->escale || (w->nnz2 > 0 && !w->eidx))) return TERN_ERR_NULL;
    if (w->ecount && (w->nnz2 < 0 || w->nnz2 > 0x7fffffff)) return TERN_ERR_SHAPE;
    const tern_status cs = run_checked(st, [&](unsigned int* f) {
        validate_codes_kernel<<<grid_for(n1, 256), 256, 0, st>>>(w->plane1, n1, f);
        if (n2) validate_codes_kernel<<<grid_for(n2, 256), 256, 0, st>>>(w->plane2, n2, f);
        // without residual rows the slot map may be absent (as tern_linear accepts); when given
        // it must hold -1 everywhere
        if (w->res_slot)
            validate_residual_kernel<<<grid_for(w->N + w->r, 256), 256, 0, st>>>(w->res_rows, w->res_slot, w->N,
                                                                                w->r, f);
    }, TERN_ERR_BAD_CODE);
    if (cs != TERN_OK || !w->ecount) return cs;
    return elem_check(*w, st);
}

extern "C" tern_status tern_device_status(tern_stream s) {
    cudaStream_t st = as_cuda(s);
    unsigned int* w = async_status_word();
    if (!w) return TERN_ERR_CUDA;
    unsigned int v = 0;
    const tern_status r = read_flag_slot(w, st, &v);
    if (r != TERN_OK) return r;
    if (v) {
        if (cudaMemsetAsync(w, 0, sizeof(unsigned int), st) != cudaSuccess) return TERN_ERR_CUDA;
        if (cudaStreamSynchronize(st) != cudaSuccess) return TERN_ERR_CUDA;
        return (v & dev::kStatusBounds) ? TERN_ERR_BOUNDS : TERN_ERR_TIMEOUT;
    }
    return TERN_OK;
}

extern "C" int tern_debug_build(void) {
#ifdef TERN_DEBUG
    return 1;
#else
    return 0;
#endif
}

extern "C" tern_status tern_residual_strip_counts(const int32_t* res_rows, int64_t r, int64_t N, uint16_t* counts) {
    if (r < 0 || N < 0 || r > N) return TERN_ERR_SHAPE;
    if ((r > 0 && !res_rows) || (N > 0 && !counts)) return TERN_ERR_NULL;
    const int64_t strips = (N + 15) / 16;
    for (int64_t j = 0; j < strips; ++j) counts[j] = 0;
    for (int64_t i = 0; i < r; ++i) {
        const int64_t n = res_rows[i];
        if (n < 0 || n >= N || (i > 0 && n <= res_rows[i - 1])) return TERN_ERR_RESIDUAL;
        ++counts[n / 16];
    }
    return TERN_OK;
}

extern "C" tern_status tern_pack_residual(const int32_t* res_rows, int64_t r, int64_t N, int32_t* res_slot,
                                          uint8_t* row_bitmap, tern_stream s) {
    if (N < 0 || r < 0 || r > N || N > (int64_t(1) << 31) - 1) return TERN_ERR_SHAPE;
    if (N == 0) return TERN_OK;
    if (!res_slot || (r > 0 && !res_rows)) return TERN_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(res_slot) & 3u) || (reinterpret_cast<uintptr_t>(res_rows) & 3u))
        return TERN_ERR_ALIGN;
    cudaStream_t st = as_cuda(s);
    return run_checked(st, [&](unsigned int* f) {
        slot_fill_kernel<<<grid_for(N, 256), 256, 0, st>>>(res_slot, N);
        if (r > 0) slot_scatter_kernel<<<grid_for(r, 256), 256, 0, st>>>(res_rows, r, N, res_slot, f);
        if (row_bitmap) bitmap_from_slots_kernel<<<grid_for((N + 7) / 8, 256), 256, 0, st>>>(res_slot, N, row_bitmap);
    }, TERN_ERR_RESIDUAL);
}

extern "C" tern_status tern_unpack_residual(const uint8_t* row_bitmap, int64_t N, int32_t* res_rows, int64_t r_cap,
                                            int64_t* r, int32_t* res_slot, tern_stream s) {
    if (N < 0 || r_cap < 0 || N > (int64_t(1) << 31) - 1) return TERN_ERR_SHAPE;
    if (!r) return TERN_ERR_NULL;
    *r = 0;
    if (N == 0) return TERN_OK;
    if (!row_bitmap) return TERN_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(res_slot) & 3u) || (reinterpret_cast<uintptr_t>(res_rows) & 3u))
        return TERN_ERR_ALIGN;
    cudaStream_t st = as_cuda(s);
    unsigned int* count = acquire_flag_slot(st);
    if (!count) return TERN_ERR_CUDA;
    const tern_status rs = run_checked(st, [&](unsigned int* f) {
        rows_from_bitmap_kernel<<<1, kRowsThreads, 0, st>>>(row_bitmap, N, res_rows, res_rows ? r_cap : 0, res_slot,
                                                            count, f);
    }, TERN_ERR_BAD_CODE);
    if (rs != TERN_OK && rs != TERN_ERR_BAD_CODE) return rs;
    unsigned int c = 0;
    const tern_status cs = read_flag_slot(count, st, &c);
    if (cs != TERN_OK) return cs;
    *r = int64_t(c);
    if (rs != TERN_OK) return rs;
    return (res_rows && int64_t(c) > r_cap) ? TERN_ERR_WORKSPACE : TERN_OK;
}

extern "C" tern_status tern_selftest_timeout(int64_t cycles, tern_stream s) {
    if (cycles < 1 || cycles > (int64_t(1) << 32)) return TERN_ERR_SHAPE;
    unsigned int* w = async_status_word();
    if (!w) return TERN_ERR_CUDA;
    selftest_timeout_kernel<<<1, 1, 0, as_cuda(s)>>>(uint64_t(cycles), w);
    return cudaGetLastError() == cudaSuccess ? TERN_OK : TERN_ERR_CUDA;
}
