// C ABI of libtern.so: argument validation and dispatch of tern_linear.
//
// tern_linear computes y = x . W^T for a ternarized W (planes T1, T2 with fp16 group-128
// scales; "Post-Training Ternarization of Qwen3-4B", arXiv 2609.01962v1, sections 4.3-4.5)
// on fp16 activations. M <= 16 (decode) runs the split-K GEMV on the packed planes; larger
// M (prefill) runs the dequantise-into-tcgen05 GEMM. Both read the packed planes directly,
// never a floating reconstruction of W (section 14: native kernels consume the ternary
// planes; section 15: a lossless native kernel).
#include <algorithm>
#include <map>
#include <mutex>
#include <vector>

#include "tern_internal.cuh"

namespace tern {

namespace {
std::mutex g_plan_mu;
std::map<std::vector<int64_t>, std::vector<int32_t>> g_plans;   // balanced splits by weights and plan
constexpr size_t kMaxPlans = 4096;
}  // namespace

bool balanced_ranges(const tern_weight* const* ws, int nw, int64_t S, int64_t P, int Sb, int nstage,
                     int seg_strips, int max_segs, int32_t* jb) {
    bool any_res = false;
    int64_t nstrips = 0;
    for (int i = 0; i < nw; ++i) {
        if (ws[i]->r > 0) {
            if (!ws[i]->res_per_strip) return false;
            any_res = true;
        }
        nstrips += (ws[i]->N + 15) / 16;
    }
    if (!any_res || P < 1 || P > kMaxBalancedGrid || nstrips != S || Sb < 1 || nstage < 1) return false;
    std::vector<int64_t> key = {S, P, Sb, nstage, seg_strips, max_segs};
    for (int i = 0; i < nw; ++i) {
        key.push_back(int64_t(reinterpret_cast<uintptr_t>(ws[i]->plane1)));
        key.push_back(int64_t(reinterpret_cast<uintptr_t>(ws[i]->res_per_strip)));
        key.push_back(ws[i]->N);
        key.push_back(ws[i]->r);
    }
    {
        std::lock_guard<std::mutex> lock(g_plan_mu);
        auto it = g_plans.find(key);
        if (it != g_plans.end()) {
            std::copy(it->second.begin(), it->second.end(), jb);
            return true;
        }
    }
    // every strip's weight and residual rows
    std::vector<int32_t> wi(size_t(S), 0), rr(size_t(S), 0);
    for (int i = 0, j = 0; i < nw; ++i)
        for (int64_t t = 0; t < (ws[i]->N + 15) / 16; ++t, ++j) {
            wi[size_t(j)] = i;
            rr[size_t(j)] = ws[i]->r > 0 ? int32_t(ws[i]->res_per_strip[t]) : 0;
        }
    auto cdiv = [](int64_t a, int64_t b) { return (a + b - 1) / b; };
    auto seg_cost = [&](int64_t nmain, int64_t rows) { return (cdiv(nmain, Sb) + cdiv(cdiv(rows, 16), Sb)) * nstage; };
    // can P ranges of cost <= T each cover the strips? (greedy, the kernel's segmentation)
    std::vector<int32_t> out(size_t(P) + 1);
    auto fill = [&](int64_t T) -> bool {
        int64_t start = 0;
        for (int64_t b = 0; b < P; ++b) {
            out[size_t(b)] = int32_t(start);
            int64_t done = 0, segs = 0, seg0 = start, smain = 0, srows = 0, end = start;
            while (end < S) {
                const bool fresh = end == start || wi[size_t(end)] != wi[size_t(seg0)] || end - seg0 >= seg_strips;
                int64_t d = done, ns = segs, s0 = seg0, m = smain, rws = srows;
                if (fresh) {
                    if (end > start) d += seg_cost(smain, srows);
                    ++ns;
                    s0 = end;
                    m = 0;
                    rws = 0;
                }
                ++m;
                rws += rr[size_t(end)];
                if (ns > max_segs || d + seg_cost(m, rws) > T) break;
                done = d;
                segs = ns;
                seg0 = s0;
                smain = m;
                srows = rws;
                ++end;
            }
            if (end == start && start < S) return false;
            start = end;
        }
        out[size_t(P)] = int32_t(S);
        return start >= S;
    };
    int64_t lo = 1, hi = int64_t(1) << 40;
    if (!fill(hi)) return false;
    while (lo < hi) {
        const int64_t mid = lo + (hi - lo) / 2;
        if (fill(mid)) hi = mid;
        else lo = mid + 1;
    }
    if (!fill(lo)) return false;
    std::copy(out.begin(), out.end(), jb);
    std::lock_guard<std::mutex> lock(g_plan_mu);
    if (g_plans.size() >= kMaxPlans) g_plans.clear();
    g_plans.emplace(std::move(key), out);
    return true;
}

int sm_count() {
    static std::mutex mu;
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    std::lock_guard<std::mutex> lock(mu);
    if (!cache[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

namespace {

constexpr int64_t kMaxRows = int64_t(1) << 22;    // grid limits of the kernels
constexpr int64_t kMaxK = int64_t(1) << 20;
constexpr int64_t kGemvMaxM = 16;

tern_status check_weight(const tern_weight* w) {
    if (!w) return TERN_ERR_NULL;
    if (w->N <= 0 || w->K <= 0 || w->K % kGroup || w->group != kGroup) return TERN_ERR_SHAPE;
    if (w->N > kMaxRows || w->K > kMaxK || w->r < 0 || w->r > w->N) return TERN_ERR_SHAPE;
    if (!w->plane1 || !w->scale1) return TERN_ERR_NULL;
    if (w->r > 0 && (!w->plane2 || !w->scale2 || !w->res_slot)) return TERN_ERR_NULL;
    if (!aligned16(w->plane1) || !aligned16(w->scale1)) return TERN_ERR_ALIGN;
    if (w->r > 0 && (!aligned16(w->plane2) || !aligned16(w->scale2) || !aligned16(w->res_slot)))
        return TERN_ERR_ALIGN;
    if (w->mu && !aligned16(w->mu)) return TERN_ERR_ALIGN;
    if (w->ecount) {
        if (w->r > 0 || w->nnz2 < 0 || w->nnz2 > 0x7fffffff || w->K / kGroup > 65535) return TERN_ERR_SHAPE;
        if (!w->ebase || !w->escale || (w->nnz2 > 0 && !w->eidx)) return TERN_ERR_NULL;
        if (!aligned16(w->ecount) || !aligned16(w->ebase) || !aligned16(w->escale) || (w->eidx && !aligned16(w->eidx)))
            return TERN_ERR_ALIGN;
    }
    return TERN_OK;
}

}  // namespace
}  // namespace tern

using namespace tern;

extern "C" size_t tern_linear_workspace_bytes(const tern_weight* w, int64_t M) {
    if (check_weight(w) != TERN_OK || M <= 0) return 0;
    const size_t b = M <= kGemvMaxM ? gemv_workspace_bytes(*w, M) : gemm_workspace_bytes(*w, M);
    return (b + 255) & ~size_t(255);
}

namespace {

bool overlap(const void* a, size_t abytes, const void* b, size_t bbytes) {
    const uintptr_t ab = reinterpret_cast<uintptr_t>(a), bb = reinterpret_cast<uintptr_t>(b);
    return ab < bb + bbytes && bb < ab + abytes;
}

tern_status linear_group(const tern_weight* const* w, int n, const tern_half* x, int64_t M, tern_half* const* y,
                         void* workspace, size_t workspace_bytes, const tern_weight* const* next, int nnext,
                         tern_stream stream) {
    if (n < 1 || n > kMaxGemvGroup || nnext < 0 || nnext > kMaxGemvGroup) return TERN_ERR_SHAPE;
    if (!w || !y || (nnext > 0 && !next)) return TERN_ERR_NULL;
    for (int i = 0; i < n; ++i) {
        const tern_status ws = check_weight(w[i]);
        if (ws != TERN_OK) return ws;
        if (w[i]->K != w[0]->K) return TERN_ERR_SHAPE;
        if ((w[i]->ecount != nullptr) != (w[0]->ecount != nullptr)) return TERN_ERR_SHAPE;
    }
    for (int j = 0; j < nnext; ++j) {
        const tern_status ns = check_weight(next[j]);
        if (ns != TERN_OK) return ns;
    }
    if (M < 0 || M > (int64_t(1) << 31)) return TERN_ERR_SHAPE;
    if (M == 0) return TERN_OK;
    if (!x) return TERN_ERR_NULL;
    if (!aligned16(x)) return TERN_ERR_ALIGN;
    size_t need = 0;
    for (int i = 0; i < n; ++i) {
        if (!y[i]) return TERN_ERR_NULL;
        if (!aligned16(y[i])) return TERN_ERR_ALIGN;
        const size_t b = tern_linear_workspace_bytes(w[i], M);
        need = b > need ? b : need;
    }
    if (need && (!workspace || workspace_bytes < need)) return TERN_ERR_WORKSPACE;
    if (workspace && !aligned16(workspace)) return TERN_ERR_ALIGN;
    // no output overlaps x or another output
    const size_t xbytes = size_t(M) * size_t(w[0]->K) * 2;
    for (int i = 0; i < n; ++i) {
        const size_t yi = size_t(M) * size_t(w[i]->N) * 2;
        if (overlap(x, xbytes, y[i], yi)) return TERN_ERR_SHAPE;
        for (int j = 0; j < i; ++j)
            if (overlap(y[j], size_t(M) * size_t(w[j]->N) * 2, y[i], yi)) return TERN_ERR_SHAPE;
    }
    cudaStream_t st = as_cuda(stream);
    const __half* xh = reinterpret_cast<const __half*>(x);
    __half* yh[kMaxGemvGroup];
    for (int i = 0; i < n; ++i) yh[i] = reinterpret_cast<__half*>(y[i]);
    if (M == 1 && decode1_supported(w, n)) return decode1_launch_group(w, n, xh, yh, next, nnext, st);
    // the multi-token kernel: from 9 tokens on, and up to 8 on launches with many strips per CTA
    // (decodem_supported); the cluster kernel otherwise (measured on the 4B and 8B layers)
    if (M >= 2 && decodem_supported(w, n, M, xh))
        return decodem_launch_group(w, n, xh, M, yh, next, nnext, st);
    if (M <= kGemvMaxM) return gemv_launch_group(w, n, xh, int(M), yh, next, nnext, st);
    for (int i = 0; i < n; ++i) {
        const tern_status s = gemm_launch(*w[i], xh, M, yh[i], workspace, st);
        if (s != TERN_OK) return s;
    }
    return TERN_OK;
}

}  // namespace

extern "C" tern_status tern_linear_group(const tern_weight* const* w, int32_t n, const tern_half* x, int64_t M,
                                         tern_half* const* y, void* workspace, size_t workspace_bytes,
                                         const tern_weight* const* next, int32_t n_next, tern_stream stream) {
    return linear_group(w, n, x, M, y, workspace, workspace_bytes, next, n_next, stream);
}

extern "C" tern_status tern_decode_ranges(const tern_weight* const* w, int32_t n, int64_t M, int32_t* ranges,
                                          int32_t max_ctas, int32_t* n_ctas, int32_t* strips_per_block,
                                          int32_t* stages_per_block) {
    if (n < 1 || n > kMaxGemvGroup || max_ctas < 1) return TERN_ERR_SHAPE;
    if (!w || !ranges || !n_ctas) return TERN_ERR_NULL;
    for (int i = 0; i < n; ++i) {
        const tern_status ws = check_weight(w[i]);
        if (ws != TERN_OK) return ws;
        if (w[i]->K != w[0]->K) return TERN_ERR_SHAPE;
        if ((w[i]->ecount != nullptr) != (w[0]->ecount != nullptr)) return TERN_ERR_SHAPE;
    }
    if (M < 1 || M > (int64_t(1) << 31)) return TERN_ERR_SHAPE;
    int Sb = 0, nstage = 0, P = 0;
    if (M == 1 && decode1_supported(w, n)) P = decode1_ranges(w, n, ranges, max_ctas, Sb, nstage);
    else if (M >= 2 && decodem_supported(w, n, M, nullptr)) P = decodem_ranges(w, n, M, ranges, max_ctas, Sb, nstage);
    if (P < 0) return TERN_ERR_SHAPE;
    *n_ctas = P;
    if (strips_per_block) *strips_per_block = Sb;
    if (stages_per_block) *stages_per_block = nstage;
    return TERN_OK;
}

extern "C" tern_status tern_linear(const tern_weight* w, const tern_half* x, int64_t M, tern_half* y,
                                   void* workspace, size_t workspace_bytes, tern_stream stream) {
    if (!w) return TERN_ERR_NULL;
    return linear_group(&w, 1, x, M, &y, workspace, workspace_bytes, nullptr, 0, stream);
}

extern "C" tern_status tern_linear_with_prefetch(const tern_weight* w, const tern_half* x, int64_t M, tern_half* y,
                                                 void* workspace, size_t workspace_bytes, const tern_weight* next,
                                                 tern_stream stream) {
    if (!w) return TERN_ERR_NULL;
    return linear_group(&w, 1, x, M, &y, workspace, workspace_bytes, next ? &next : nullptr, next ? 1 : 0, stream);
}
