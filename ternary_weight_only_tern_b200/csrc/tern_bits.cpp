// Bit accounting of one ternarized tensor (host only, exact integers).
//
// The pages separate three quantities ("Post-Training Ternarization of Qwen3-4B",
// arXiv 2609.01962v1, sections 3.2, 4.4 and 7.1; the Qwen3-8B scale-up paper,
// arXiv 2609.09240, effective-bit discussion): the information rate of the adaptive
// planes (1.641 bits per weight measured, against log2 3 = 1.585 for one plane),
// which counts log2 3 per plane symbol with a fraction f2 of weights carrying a second
// plane; and what a file or an execution buffer actually holds. This function reports
// all three for the row-subset form and for the element-level second plane.
#include <math.h>

#include "../../include/tern.h"

extern "C" tern_status tern_bits(int64_t N, int64_t K, int64_t r, int32_t group, tern_bits_report* out) {
    if (!out) return TERN_ERR_NULL;
    if (N <= 0 || K <= 0 || group != 128 || K % group || r < 0 || r > N) return TERN_ERR_SHAPE;
    // 2^63 guard for the largest product below, 2*(N+r)*K + ...
    if (N > (int64_t(1) << 40) || K > (int64_t(1) << 20)) return TERN_ERR_SHAPE;
    const uint64_t n = static_cast<uint64_t>(N), k = static_cast<uint64_t>(K), rr = static_cast<uint64_t>(r);
    const uint64_t G = k / static_cast<uint64_t>(group);
    const uint64_t plane_rows = n + rr;
    const uint64_t header_bits = 512;                  // 64-byte container header
    const uint64_t store_row_bytes = (k + 4) / 5;      // 5 trits per base-3 byte
    const uint64_t bitmap_bits = 8 * ((n + 7) / 8);    // residual-row bitmap, whole bytes
    out->weights = n * k;
    out->plane_trits = plane_rows * k;
    out->store_bits = 8 * plane_rows * store_row_bytes + 16 * plane_rows * G + bitmap_bits + header_bits;
    out->exec_bits = 2 * plane_rows * k + 16 * plane_rows * G + 32 * n + header_bits;
    const double w = static_cast<double>(out->weights);
    out->bpw_info = log2(3.0) * static_cast<double>(out->plane_trits) / w;
    out->bpw_store = static_cast<double>(out->store_bits) / w;
    out->bpw_exec = static_cast<double>(out->exec_bits) / w;
    return TERN_OK;
}

extern "C" tern_status tern_bits_offset(int64_t N, int64_t K, int64_t r, int32_t group, tern_bits_report* out) {
    const tern_status st = tern_bits(N, K, r, group, out);
    if (st != TERN_OK) return st;
    const uint64_t offset_bits = 16 * static_cast<uint64_t>(N) * static_cast<uint64_t>(K / group);
    out->store_bits += offset_bits;
    out->exec_bits += offset_bits;
    const double w = static_cast<double>(out->weights);
    out->bpw_store = static_cast<double>(out->store_bits) / w;
    out->bpw_exec = static_cast<double>(out->exec_bits) / w;
    return TERN_OK;
}

extern "C" tern_status tern_bits_elem(int64_t N, int64_t K, int64_t masked, int64_t nnz2, int32_t group,
                                      int32_t offset, tern_bits_report* out) {
    if (!out) return TERN_ERR_NULL;
    if (N <= 0 || K <= 0 || group != 128 || K % group) return TERN_ERR_SHAPE;
    if (N > (int64_t(1) << 40) || K > (int64_t(1) << 20) || N > (int64_t(1) << 62) / K) return TERN_ERR_SHAPE;
    if (masked < 0 || masked > N * K || nnz2 < 0 || nnz2 > masked) return TERN_ERR_SHAPE;
    const uint64_t n = static_cast<uint64_t>(N), k = static_cast<uint64_t>(K);
    const uint64_t G = k / static_cast<uint64_t>(group);
    const uint64_t blocks = (n + 63) / 64;             // ebase: one entry per (group, 64-row block), + 1
    const uint64_t header_bits = 512;
    const uint64_t store_row_bytes = (k + 4) / 5;
    const uint64_t elem_bits = 8 * G * n + 32 * (G * blocks + 1) + 8 * static_cast<uint64_t>(nnz2) + 16 * n * G;
    out->weights = n * k;
    out->plane_trits = n * k + static_cast<uint64_t>(masked);
    out->store_bits = 8 * n * store_row_bytes + 16 * n * G + elem_bits + header_bits;
    out->exec_bits = 2 * n * k + 16 * n * G + elem_bits + header_bits;
    if (offset) {
        out->store_bits += 16 * n * G;
        out->exec_bits += 16 * n * G;
    }
    const double w = static_cast<double>(out->weights);
    out->bpw_info = log2(3.0) * static_cast<double>(out->plane_trits) / w;
    out->bpw_store = static_cast<double>(out->store_bits) / w;
    out->bpw_exec = static_cast<double>(out->exec_bits) / w;
    return TERN_OK;
}

extern "C" const char* tern_status_string(tern_status s) {
    switch (s) {
        case TERN_OK: return "ok";
        case TERN_ERR_NULL: return "null pointer";
        case TERN_ERR_SHAPE: return "invalid shape";
        case TERN_ERR_ALIGN: return "pointer not 16-byte aligned";
        case TERN_ERR_BAD_TRIT: return "input trit outside {-1, 0, +1}";
        case TERN_ERR_BAD_CODE: return "invalid packed code";
        case TERN_ERR_RESIDUAL: return "inconsistent residual-row metadata";
        case TERN_ERR_WORKSPACE: return "workspace too small";
        case TERN_ERR_CUDA: return "CUDA error";
        case TERN_ERR_TIMEOUT: return "device wait timed out";
        case TERN_ERR_ELEM: return "inconsistent element-plane metadata";
        case TERN_ERR_BOUNDS: return "a device-side bounds check of the debug build failed";
    }
    return "unknown status";
}

extern "C" int tern_version(void) { return 100; }
