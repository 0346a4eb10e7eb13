// Internal declarations shared by the libtern.so translation units (not installed).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/tern.h"

namespace tern {

constexpr int kGroup = 128;          // K columns per scale group
constexpr int kCodesPerWord = 16;    // 2-bit codes per uint32 of the exec plane
constexpr int kWordsPerGroup = kGroup / kCodesPerWord;
constexpr int kTritsPerByte = 5;     // base-3 storage

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline cudaStream_t as_cuda(tern_stream s) { return reinterpret_cast<cudaStream_t>(s); }

// Device-side status words for the synchronous pack/unpack/validate calls (tern_pack.cu).
// Returns a device pointer to a zeroed slot, or nullptr on a CUDA error.
unsigned int* acquire_flag_slot(cudaStream_t stream);
tern_status read_flag_slot(unsigned int* slot, cudaStream_t stream, unsigned int* value);
// Device address of this device's sticky status word for asynchronous kernels (bounded waits
// that ran out set it); nullptr on a CUDA error.
unsigned int* async_status_word();

// Decode GEMV on a thread-block cluster per 64-row block (tern_gemv.cu), M in [1, 16], for
// 1..kMaxGemvGroup weights of the same K that share x (one launch; output i is ys[i]). The
// launch also prefetches the planes, scales and slot maps of the `nnext` weights `next` into L2.
constexpr int kMaxGemvGroup = 4;
tern_status gemv_launch_group(const tern_weight* const* ws, int nw, const __half* x, int M, __half* const* ys,
                              const tern_weight* const* next, int nnext, cudaStream_t stream);
size_t gemv_workspace_bytes(const tern_weight& w, int64_t M);

// Decode GEMV for one token on a persistent, warp-specialised grid (tern_decode1.cu): row-level
// residual planes and offsets, K % 512 == 0; decode1_supported tells whether it takes the call.
// The persistent decode kernels' split of a launch's S strips (the weights' strips in order)
// among P CTAs, balanced by what each CTA walks: per segment (at most seg_strips strips of one
// weight, starting at the CTA's first strip), ceil(main strips / Sb) + ceil(residual strips / Sb)
// blocks of nstage stages, a segment's residual strips being ceil(its residual rows / 16); at
// most max_segs segments per CTA. CTA b takes strips [jb[b], jb[b + 1]). False (the caller
// splits evenly) when a weight with residual rows has no res_per_strip, no weight has residual
// rows, or P > kMaxBalancedGrid. Cached per weights and plan.
constexpr int kMaxBalancedGrid = 192;
bool balanced_ranges(const tern_weight* const* ws, int nw, int64_t S, int64_t P, int Sb, int nstage,
                     int seg_strips, int max_segs, int32_t* jb);
constexpr int64_t kMaxLaunchStrips = int64_t(1) << 24;   // 16-row strips of one persistent decode launch
bool decode1_supported(const tern_weight* const* ws, int nw);
// The CTA strip ranges (jb[0..P]) and plan (strips per block, stages per block) the one-token
// launch would use; P, or -1 when P > max_ctas or there is no layout.
int decode1_ranges(const tern_weight* const* ws, int nw, int32_t* jb, int max_ctas, int& Sb, int& nstage);
tern_status decode1_launch_group(const tern_weight* const* ws, int nw, const __half* x, __half* const* ys,
                                 const tern_weight* const* next, int nnext, cudaStream_t stream);

// Decode GEMV for 2..16 tokens on the same persistent grid (tern_decodem.cu): the tokens are
// the MMA's columns, x streams beside the weights; decodem_supported tells whether it takes the call.
constexpr int64_t kDecodemMinM = 9;        // from this M on the multi-token kernel takes every launch
constexpr int64_t kDecodemMinStrips = 10;  // below it, from kDecodemStripsMinM tokens, launches of at
constexpr int64_t kDecodemStripsMinM = 4;  // least kDecodemMinStrips strips per CTA (measured: at 4 tokens the
                                            // 8B stack 2239 against 2420 us per step, at 2 tokens 2095 against 2080)
bool decodem_supported(const tern_weight* const* ws, int nw, int64_t M, const void* x);
int decodem_ranges(const tern_weight* const* ws, int nw, int64_t M, int32_t* jb, int max_ctas, int& Sb,
                   int& nstage);
tern_status decodem_launch_group(const tern_weight* const* ws, int nw, const __half* x, int64_t M, __half* const* ys,
                                 const tern_weight* const* next, int nnext, cudaStream_t stream);

// Prefill GEMM on tcgen05 (tern_gemm_sm100.cu), M > 16.
tern_status gemm_launch(const tern_weight& w, const __half* x, int64_t M, __half* y, void* workspace,
                        cudaStream_t stream);
size_t gemm_workspace_bytes(const tern_weight& w, int64_t M);

// Consistency of a descriptor's element plane (tern_elem.cu): TERN_OK or TERN_ERR_ELEM.
tern_status elem_check(const tern_weight& w, cudaStream_t stream);

constexpr int kElemBlock = 64;       // rows per ebase entry of the element plane

int sm_count();   // of the current device, cached per device

}  // namespace tern
