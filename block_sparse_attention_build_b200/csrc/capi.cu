// C ABI of the forward pass: argument checks, TMA descriptors, kernel choice
// and launch, the host-buffer variant, and the device status word.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/sparse_attn.h"
#include "fwd_sm100.cuh"
#include "runtime.h"
#include "stride_sm100.cuh"
#include "tma_host.h"

namespace sa {
namespace {

constexpr long long kDefaultTimeout = 2000000000LL;  // SM cycles, about one second
constexpr int kMaxDevices = 64;

std::mutex g_mu;
int32_t* g_status[kMaxDevices] = {};  // one status word per device, allocated on first use
int32_t g_debug_flags = 0;
long long g_timeout = kDefaultTimeout;

// The device status word of the current device, allocated once.
int status_word(int32_t** out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SA_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_status[dev]) {
        // first use on this device: allocate and clear the word, and wait for
        // the clear, so that no stream's kernel can see it before it is zero
        int32_t* p = nullptr;
        if (cudaMalloc(&p, sizeof(int32_t)) != cudaSuccess) return SA_ERR_CUDA;
        if (cudaMemset(p, 0, sizeof(int32_t)) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
            cudaFree(p);
            return SA_ERR_CUDA;
        }
        g_status[dev] = p;
    }
    *out = g_status[dev];
    return SA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Number of SMs of the current device (cached).
int sm_count()
{
    static int counts[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
    if (!counts[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        counts[dev] = n;
    }
    return counts[dev];
}

template <int D, int BN, bool MULTI>
int launch(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mo, const FwdParams& p,
           const HeadPatterns& hp, int grid, cudaStream_t stream)
{
    using C = FwdCfg<D, BN>;
    auto kern = fwd_kernel<D, BN, MULTI>;
    static bool attr_set[kMaxDevices] = {};  // per instantiation and device
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SA_ERR_CUDA;
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess)
            return SA_ERR_CUDA;
        // the warpgroups' register split must fit what the kernel is launched with
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return SA_ERR_CUDA;
        if (fa.numRegs * kThreads < kRegSplitTotal) return SA_ERR_UNSUPPORTED;
        attr_set[dev] = true;
    }
    kern<<<grid, kThreads, C::kSmemBytes, stream>>>(mq, mk, mv, mo, p, hp);
    return cudaGetLastError() == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

template <bool MULTI>
int launch_any(int D, int block, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
               const CUtensorMap& mo, const FwdParams& p, const HeadPatterns& hp, int g, cudaStream_t st)
{
    if (D == 128 && block == 128) return launch<128, 128, MULTI>(mq, mk, mv, mo, p, hp, g, st);
    if (D == 64 && block == 128) return launch<64, 128, MULTI>(mq, mk, mv, mo, p, hp, g, st);
    if (D == 128 && block == 64) return launch<128, 64, MULTI>(mq, mk, mv, mo, p, hp, g, st);
    return launch<64, 64, MULTI>(mq, mk, mv, mo, p, hp, g, st);
}

// SA_OK, SA_ERR_INVALID_ARG (a negative field) or SA_ERR_UNSUPPORTED (a form
// the library does not build: causal not 0 or 1, a stride without causality
// or with stripes).
int pattern_status(const sa_pattern& pt)
{
    if (pt.window < -1 || pt.sinks < 0 || pt.stride < 0 || pt.n_global < 0 || pt.area < 0 || pt.summary < 0)
        return SA_ERR_INVALID_ARG;
    if (pt.summary > 0 && pt.area == 0) return SA_ERR_INVALID_ARG;
    if (pt.causal != 0 && pt.causal != 1) return SA_ERR_UNSUPPORTED;
    if (pt.stride > 0 && (pt.causal == 0 || pt.area > 0)) return SA_ERR_UNSUPPORTED;
    return SA_OK;
}

// Forms beyond the causal band / sinks / stride / global rules: the kernel
// instantiation with a pattern table masks them.
bool general_form(const sa_pattern& pt) { return pt.causal == 0 || pt.area > 0; }

// Window and stripe clipped to the sequence (same allowed set), so that the
// kernels' q - kv +- window and stripe bounds stay inside int32.
int32_t clip_to(int32_t v, int32_t N) { return v > N ? N : v; }

// Pass 2 of the stride-aware path: the residual stride pairs in the grouped
// order (PatternRef mode 1).
struct ResidualStride {
    int32_t n;       // group length N / stride
    int32_t shift;   // floor(window / stride) + 1 (0 without a band)
    int32_t col_lo;  // max(sinks, n_global)
    int32_t stride;
    bool view;       // Q, K, V, O are token-order tensors read and written through grouped-view maps
};

// Grouped-view maps need the group length to be a multiple of the tile
// heights (128 query rows, `block` kv rows): a tile never spans two groups.
bool grouped_view_ok(int32_t n, int32_t block) { return n % kBM == 0 && n % block == 0; }

// The forward pass behind sparse_attn_fwd (one pattern: n_patterns = 1,
// head_pattern = null), sparse_attn_fwd_heads (a pattern per query head) and
// pass 2 of sparse_attn_fwd_stride (rs non-null).
int fwd_impl(const void* Q, const void* K, const void* V, const sa_block_mask* masks, const sa_pattern* patterns,
             int32_t n_patterns, const int32_t* head_pattern, const sa_shape* shape, float scale, void* O, float* LSE,
             void* stream, const ResidualStride* rs = nullptr)
{
    if (!masks || !patterns || !shape) return SA_ERR_INVALID_ARG;
    const bool per_head = head_pattern != nullptr;
    if (n_patterns < 1 || n_patterns > (per_head ? kMaxPatterns : 1)) return SA_ERR_INVALID_ARG;
    bool multi = per_head || rs != nullptr;  // general forms also take the pattern-table kernel
    for (int i = 0; i < n_patterns; i++) multi = multi || general_form(patterns[i]);
    const sa_block_mask* mask = &masks[0];
    const sa_pattern* pattern = &patterns[0];
    const sa_shape s = *shape;
    if (s.B < 0 || s.Hq < 0 || s.Hkv < 0 || s.N < 0 || s.D <= 0) return SA_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !std::isfinite(scale)) return SA_ERR_INVALID_ARG;
    for (int i = 0; i < n_patterns; i++)
        if (int rc = pattern_status(patterns[i])) return rc;
    if (s.D != 64 && s.D != 128) return SA_ERR_UNSUPPORTED;
    if (mask->block != 64 && mask->block != 128) return SA_ERR_UNSUPPORTED;
    for (int i = 1; i < n_patterns; i++)
        if (masks[i].block != mask->block) return SA_ERR_MASK_MISMATCH;
    if (multi && s.Hq > kMaxHeadsMulti) return SA_ERR_UNSUPPORTED;
    if (per_head)
        for (int h = 0; h < s.Hq; h++)
            if (head_pattern[h] < 0 || head_pattern[h] >= n_patterns) return SA_ERR_INVALID_ARG;
    if (s.B == 0 || s.Hq == 0 || s.N == 0) return SA_OK;  // nothing to compute
    if (s.Hkv <= 0 || s.Hq % s.Hkv != 0) return SA_ERR_UNSUPPORTED;
    const int64_t T = (int64_t(s.N) + mask->block - 1) / mask->block;
    for (int i = 0; i < n_patterns; i++) {
        if (masks[i].n_q_tiles != T || masks[i].n_kv_tiles != T) return SA_ERR_MASK_MISMATCH;
        if (!masks[i].kv_count || !masks[i].kv_index || !masks[i].kv_full) return SA_ERR_INVALID_ARG;
    }

    if (T > kMaxTiles) return SA_ERR_UNSUPPORTED;
    if (!Q || !K || !V || !O || !LSE) return SA_ERR_INVALID_ARG;
    // LSE is written one fp32 at a time: 4-byte alignment is enough
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || (reinterpret_cast<uintptr_t>(LSE) & 3u))
        return SA_ERR_MISALIGNED;
    for (int i = 0; i < n_patterns; i++)  // the first CUDA call of the path
        if (int rc = check_device_mask(&masks[i])) return rc;
    const int64_t n_qtiles = (int64_t(s.N) + kBM - 1) / kBM;
    const int64_t group = s.Hq / s.Hkv;
    // work units: two 128-row query tiles that share a key/value head
    const int64_t pairs = group >= 2 ? (group + 1) / 2 : (n_qtiles + 1) / 2;
    const int64_t n_units = group >= 2 ? n_qtiles * s.B * s.Hkv * pairs : pairs * s.B * s.Hq;
    if (n_units > INT32_MAX || int64_t(s.B) * s.Hq > INT32_MAX) return SA_ERR_UNSUPPORTED;
    const int n_sm = sm_count();
    if (n_sm <= 0) return SA_ERR_CUDA;
    int32_t debug_flags = 0;
    long long timeout = 0;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        timeout = g_timeout;
        debug_flags = g_debug_flags;
    }
    int64_t n_whole = 0, n_items = 0;
    plan_items(n_units, n_sm, (debug_flags & kDebugSplitAll) != 0, &n_whole, &n_items);
    if (n_items > INT32_MAX) return SA_ERR_UNSUPPORTED;
    const int64_t grid = n_items < n_sm ? n_items : n_sm;

    int32_t* status = nullptr;
    if (int rc = status_word(&status)) return rc;

    CUtensorMap mq, mk, mv, mo;
    const uint32_t bn = static_cast<uint32_t>(mask->block);
    const bool view = rs && rs->view;
    if (view) {
        const uint64_t sg = static_cast<uint64_t>(rs->stride);
        if (!make_map_bf16_grouped(&mq, Q, s.D, s.N, uint64_t(s.B) * s.Hq, sg, kBM) ||
            !make_map_bf16_grouped(&mk, K, s.D, s.N, uint64_t(s.B) * s.Hkv, sg, bn) ||
            !make_map_bf16_grouped(&mv, V, s.D, s.N, uint64_t(s.B) * s.Hkv, sg, bn) ||
            !make_map_bf16_grouped(&mo, O, s.D, s.N, uint64_t(s.B) * s.Hq, sg, bn))
            return SA_ERR_CUDA;
    } else if (!make_map_bf16_3d(&mq, Q, s.D, s.N, uint64_t(s.B) * s.Hq, kBM) ||
               !make_map_bf16_3d(&mk, K, s.D, s.N, uint64_t(s.B) * s.Hkv, bn) ||
               !make_map_bf16_3d(&mv, V, s.D, s.N, uint64_t(s.B) * s.Hkv, bn) ||
               !make_map_bf16_3d(&mo, O, s.D, s.N, uint64_t(s.B) * s.Hq, bn)) {
        return SA_ERR_CUDA;
    }

    FwdParams p;
    p.kv_count = mask->kv_count;
    p.kv_index = mask->kv_index;
    p.kv_full = mask->kv_full;
    p.T = static_cast<int32_t>(T);
    p.N = s.N;
    p.B = s.B;
    p.Hq = s.Hq;
    p.Hkv = s.Hkv;
    p.group = s.Hq / s.Hkv;
    p.n_qtiles = static_cast<int32_t>(n_qtiles);
    p.n_units = static_cast<int32_t>(n_units);
    p.n_whole = static_cast<int32_t>(n_whole);
    p.n_items = static_cast<int32_t>(n_items);
    p.pairs = static_cast<int32_t>(pairs);
    p.window = clip_to(pattern->window, s.N);
    p.sinks = pattern->sinks;
    p.stride = pattern->stride;
    p.n_global = pattern->n_global;
    p.scale_log2 = scale * 1.44269504088896340736f;
    p.O = static_cast<__nv_bfloat16*>(O);
    p.LSE = LSE;
    p.status = status;
    p.timeout = timeout;
    p.debug_flags = debug_flags;
    {
        sa_block_mask_fields f{T, 0, 0};  // the longest row and the live tiles over all patterns
        for (int i = 0; i < n_patterns; i++) {
            f.n_live = masks[i].n_live > f.n_live ? masks[i].n_live : f.n_live;
            f.max_per_row = masks[i].max_per_row > f.max_per_row ? masks[i].max_per_row : f.max_per_row;
        }
        p.snake = snake_order(f);
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int g = static_cast<int>(grid);
    HeadPatterns hp{};
    hp.grp_n = view ? rs->n : 0;
    hp.grp_s = view ? rs->stride : 0;
    if (!multi) return launch_any<false>(s.D, mask->block, mq, mk, mv, mo, p, hp, g, st);
    for (int i = 0; i < n_patterns; i++) {
        hp.pat[i].kv_count = masks[i].kv_count;
        hp.pat[i].kv_index = masks[i].kv_index;
        hp.pat[i].kv_full = masks[i].kv_full;
        hp.pat[i].window = clip_to(patterns[i].window, s.N);
        hp.pat[i].sinks = patterns[i].sinks;
        hp.pat[i].stride = patterns[i].stride;
        hp.pat[i].n_global = patterns[i].n_global;
        hp.pat[i].causal = patterns[i].causal;
        hp.pat[i].area = clip_to(patterns[i].area, s.N);
        hp.pat[i].summary = patterns[i].summary < patterns[i].area ? patterns[i].summary : patterns[i].area;
        hp.pat[i].mode = 0;
    }
    if (rs) {
        hp.pat[0].mode = 1;
        hp.pat[0].area = rs->n;
        hp.pat[0].shift = rs->shift;
        hp.pat[0].col_lo = rs->col_lo;
        hp.pat[0].stride = rs->stride;
    }
    for (int h = 0; h < s.Hq; h++) hp.head[h] = per_head ? static_cast<uint8_t>(head_pattern[h]) : 0;
    return launch_any<true>(s.D, mask->block, mq, mk, mv, mo, p, hp, g, st);
}

}  // namespace

int device_status_word(int32_t** out) { return status_word(out); }

long long wait_limit_cycles()
{
    std::lock_guard<std::mutex> lk(g_mu);
    return g_timeout;
}

int32_t debug_flags()
{
    std::lock_guard<std::mutex> lk(g_mu);
    return g_debug_flags;
}

int check_host_mask(const sa_block_mask* m, int64_t T)
{
    if (!m || !m->kv_count || !m->kv_index || !m->kv_full) return SA_ERR_INVALID_ARG;
    for (int64_t i = 0; i < T; i++) {
        const int32_t c = m->kv_count[i];
        if (c < 0 || c > T) return SA_ERR_INVALID_ARG;
        const int32_t* idx = m->kv_index + i * T;
        const uint8_t* full = m->kv_full + i * T;
        int32_t prev = -1;
        for (int32_t e = 0; e < c; e++) {
            if (idx[e] <= prev || idx[e] >= T || full[e] > 1) return SA_ERR_INVALID_ARG;
            prev = idx[e];
        }
    }
    return SA_OK;
}

int device_sm_count() { return sm_count(); }

int check_device_mask(const sa_block_mask* m)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SA_ERR_CUDA;
    const void* arrays[3] = {m->kv_count, m->kv_index, m->kv_full};
    for (const void* a : arrays) {
        cudaPointerAttributes at;
        if (cudaPointerGetAttributes(&at, a) != cudaSuccess) {
            (void)cudaGetLastError();
            return SA_ERR_INVALID_ARG;
        }
        const bool ok = (at.type == cudaMemoryTypeDevice && at.device == dev) || at.type == cudaMemoryTypeManaged ||
                        at.type == cudaMemoryTypeHost;
        if (!ok) return SA_ERR_INVALID_ARG;
    }
    return SA_OK;
}

}  // namespace sa

extern "C" int sparse_attn_fwd(const void* Q, const void* K, const void* V, const sa_block_mask* mask,
                               const sa_pattern* pattern, const sa_shape* shape, float scale, void* O, float* LSE,
                               void* stream)
{
    return sa::fwd_impl(Q, K, V, mask, pattern, 1, nullptr, shape, scale, O, LSE, stream);
}

extern "C" int sparse_attn_fwd_heads(const void* Q, const void* K, const void* V, const sa_block_mask* masks,
                                     const sa_pattern* patterns, int32_t n_patterns, const int32_t* head_pattern,
                                     const sa_shape* shape, float scale, void* O, float* LSE, void* stream)
{
    if (!head_pattern) return SA_ERR_INVALID_ARG;
    return sa::fwd_impl(Q, K, V, masks, patterns, n_patterns, head_pattern, shape, scale, O, LSE, stream);
}

namespace sa {
namespace {

struct StrideLayout {
    size_t q, k, v, o2, l1, l2, total;  // byte offsets, each 256-aligned
};

StrideLayout stride_layout(const sa_shape& s)
{
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    const size_t qb = size_t(s.B) * s.Hq * s.N * s.D * 2, kvb = size_t(s.B) * s.Hkv * s.N * s.D * 2;
    const size_t lb = size_t(s.B) * s.Hq * s.N * 4;
    StrideLayout w;
    w.q = 0;
    w.k = w.q + up(qb);
    w.v = w.k + up(kvb);
    w.o2 = w.v + up(kvb);
    w.l1 = w.o2 + up(qb);
    w.l2 = w.l1 + up(lb);
    w.total = w.l2 + up(lb);
    return w;
}

unsigned grid_for(int64_t items)
{
    const int n_sm = sm_count();
    int64_t g = (items + 255) / 256;
    const int64_t cap = int64_t(n_sm > 0 ? n_sm : 148) * 16;
    return static_cast<unsigned>(g < cap ? (g > 0 ? g : 1) : cap);
}

template <int D>
int stride_run(const void* Q, const void* K, const void* V, const sa_block_mask* pass1, const sa_block_mask* pass2,
               const sa_pattern& pt, const sa_shape& s, float scale, void* O, float* LSE, uint8_t* ws,
               cudaStream_t st)
{
    const StrideLayout L = stride_layout(s);
    const int n = s.N / pt.stride;
    constexpr int U = D * 2 / 16;
    const int64_t qp = int64_t(s.B) * s.Hq, kp = int64_t(s.B) * s.Hkv;
    // pass 2 reads and writes the token-order tensors through grouped-view maps
    // when the group length fits the tiles; else through grouped copies
    const bool view = grouped_view_ok(n, pass2->block);
    if (!view) {
        group_by_residue_kernel<D><<<grid_for(qp * s.N * U), 256, 0, st>>>(
            static_cast<const uint4*>(Q), reinterpret_cast<uint4*>(ws + L.q), qp, s.N, pt.stride, n);
        group_by_residue_kernel<D><<<grid_for(kp * s.N * U), 256, 0, st>>>(
            static_cast<const uint4*>(K), reinterpret_cast<uint4*>(ws + L.k), kp, s.N, pt.stride, n);
        group_by_residue_kernel<D><<<grid_for(kp * s.N * U), 256, 0, st>>>(
            static_cast<const uint4*>(V), reinterpret_cast<uint4*>(ws + L.v), kp, s.N, pt.stride, n);
        if (cudaGetLastError() != cudaSuccess) return SA_ERR_CUDA;
    }
    // pass 1: the pattern without its stride, token order; O holds O1, L1 in the workspace
    sa_pattern p1 = pt;
    p1.stride = 0;
    float* l1 = reinterpret_cast<float*>(ws + L.l1);
    if (int rc = fwd_impl(Q, K, V, pass1, &p1, 1, nullptr, &s, scale, O, l1, st)) return rc;
    // pass 2: the residual stride pairs, grouped order
    ResidualStride rs;
    rs.n = n;
    rs.shift = pt.window >= 0 ? (pt.window > s.N ? s.N : pt.window) / pt.stride + 1 : 0;
    rs.col_lo = pt.sinks > pt.n_global ? pt.sinks : pt.n_global;
    rs.stride = pt.stride;
    rs.view = view;
    float* l2 = reinterpret_cast<float*>(ws + L.l2);
    const void* q2 = view ? Q : static_cast<const void*>(ws + L.q);
    const void* k2 = view ? K : static_cast<const void*>(ws + L.k);
    const void* v2 = view ? V : static_cast<const void*>(ws + L.v);
    if (int rc = fwd_impl(q2, k2, v2, pass2, &pt, 1, nullptr, &s, scale, ws + L.o2, l2, st, &rs)) return rc;
    // with the grouped view pass 2's O and LSE are already in token order
    merge_passes_kernel<D><<<grid_for(qp * s.N * U), 256, 0, st>>>(
        static_cast<__nv_bfloat16*>(O), LSE, reinterpret_cast<const __nv_bfloat16*>(ws + L.o2), l1, l2, qp, s.N,
        view ? 1 : pt.stride, view ? s.N : n);
    return cudaGetLastError() == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

}  // namespace
}  // namespace sa

extern "C" int sparse_attn_fwd_stride_workspace(const sa_shape* shape, size_t* bytes)
{
    if (!shape || !bytes) return SA_ERR_INVALID_ARG;
    const sa_shape s = *shape;
    if (s.B < 0 || s.Hq < 0 || s.Hkv < 0 || s.N < 0 || s.D <= 0) return SA_ERR_INVALID_ARG;
    *bytes = sa::stride_layout(s).total;
    return SA_OK;
}

extern "C" int sparse_attn_fwd_stride(const void* Q, const void* K, const void* V, const sa_block_mask* pass1,
                                      const sa_block_mask* pass2, const sa_pattern* pattern, const sa_shape* shape,
                                      float scale, void* O, float* LSE, void* workspace, size_t workspace_bytes,
                                      void* stream)
{
    if (!pass1 || !pass2 || !pattern || !shape) return SA_ERR_INVALID_ARG;
    const sa_pattern pt = *pattern;
    const sa_shape s = *shape;
    if (int rc = sa::pattern_status(pt)) return rc;
    if (pt.causal != 1 || pt.stride <= 0 || pt.area != 0) return SA_ERR_UNSUPPORTED;
    if (s.B < 0 || s.Hq < 0 || s.Hkv < 0 || s.N < 0 || s.D <= 0) return SA_ERR_INVALID_ARG;
    if (s.D != 64 && s.D != 128) return SA_ERR_UNSUPPORTED;
    if (s.B == 0 || s.Hq == 0 || s.N == 0) return SA_OK;
    if (s.N % pt.stride != 0) return SA_ERR_UNSUPPORTED;  // groups of equal length
    if (pass1->block != pass2->block) return SA_ERR_MASK_MISMATCH;
    if (!workspace || !Q || !K || !V || !O || !LSE) return SA_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return SA_ERR_MISALIGNED;
    if (!sa::aligned16(Q) || !sa::aligned16(K) || !sa::aligned16(V) || !sa::aligned16(O) || !sa::aligned16(LSE))
        return SA_ERR_MISALIGNED;
    if (workspace_bytes < sa::stride_layout(s).total) return SA_ERR_BUFFER_TOO_SMALL;
    // the passes check shapes and masks themselves before launching
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    if (s.D == 128) return sa::stride_run<128>(Q, K, V, pass1, pass2, pt, s, scale, O, LSE, ws, st);
    return sa::stride_run<64>(Q, K, V, pass1, pass2, pt, s, scale, O, LSE, ws, st);
}

namespace sa {
namespace {

// The host-buffer path works in chunks of whole kv heads (flattened over batch
// and head, index b * Hkv + h): a chunk's Q, K, V, O and LSE are one
// contiguous byte range of each tensor, so each moves with one copy, and chunk
// c + 1's inputs cross the bus while chunk c computes and chunk c - 1's
// outputs come back.  Chunks halve in size (half the heads, then half of the
// rest, ...): few copies, and only the last, one-head chunk's outputs are
// left to copy back once all inputs are in.
constexpr int kHostChunks = 16;

// Head boundaries of the chunks: first[0] = 0 < first[1] < ... < first[n] = heads.
int host_chunks(int64_t heads, int64_t* first)
{
    int n = 0;
    first[0] = 0;
    int64_t done = 0;
    while (done < heads) {
        const int64_t rest = heads - done;
        const int64_t take = (n == kHostChunks - 1) ? rest : (rest / 2 > 0 ? rest / 2 : 1);
        done += take;
        first[++n] = done;
    }
    return n;
}

struct HostLayout {
    size_t count, index, full, q, k, v, o, lse, total;  // byte offsets, each 256-aligned
};

HostLayout host_layout(const sa_shape& s)
{
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    // the mask copy is sized for the smaller tile (64), which has more tiles
    const size_t T = (size_t(s.N) + 63) / 64;
    const size_t qb = size_t(s.B) * s.Hq * s.N * s.D * 2, kvb = size_t(s.B) * s.Hkv * s.N * s.D * 2;
    HostLayout L;
    L.count = 0;
    L.index = L.count + up(T * 4);
    L.full = L.index + up(T * T * 4);
    L.q = L.full + up(T * T);
    L.k = L.q + up(qb);
    L.v = L.k + up(kvb);
    L.o = L.v + up(kvb);
    L.lse = L.o + up(qb);
    L.total = L.lse + up(size_t(s.B) * s.Hq * s.N * 4);
    return L;
}

// Per device: the streams the chunks' copies and kernels run on, and the
// events that order them (created on first use, kept until exit).
struct HostStreams {
    cudaStream_t in = nullptr, comp = nullptr, out = nullptr;
    cudaEvent_t start = nullptr, done = nullptr;
    cudaEvent_t comp_done = nullptr;  // the previous call's last kernel (its inputs are free after it)
    cudaEvent_t landed[kHostChunks] = {}, computed[kHostChunks] = {};
    // Pinned staging of the block mask: a copy from pageable memory would first
    // wait for its stream to drain, which would hold the host until the previous
    // call's kernels are done.  Reused once the previous call's copy out of it is.
    uint8_t* stage = nullptr;
    size_t stage_bytes = 0;
    cudaEvent_t staged = nullptr;
};
HostStreams g_host[kMaxDevices];
std::mutex g_host_mu[kMaxDevices];

int host_streams(int dev, HostStreams** out)
{
    HostStreams& h = g_host[dev];
    if (!h.in) {
        const unsigned ef = cudaEventDisableTiming;
        if (cudaStreamCreateWithFlags(&h.comp, cudaStreamNonBlocking) != cudaSuccess ||
            cudaStreamCreateWithFlags(&h.out, cudaStreamNonBlocking) != cudaSuccess ||
            cudaEventCreateWithFlags(&h.start, ef) != cudaSuccess || cudaEventCreateWithFlags(&h.done, ef) != cudaSuccess ||
            cudaEventCreateWithFlags(&h.comp_done, ef) != cudaSuccess ||
            cudaEventCreateWithFlags(&h.staged, ef) != cudaSuccess)
            return SA_ERR_CUDA;
        for (int c = 0; c < kHostChunks; c++)
            if (cudaEventCreateWithFlags(&h.landed[c], ef) != cudaSuccess ||
                cudaEventCreateWithFlags(&h.computed[c], ef) != cudaSuccess)
                return SA_ERR_CUDA;
        if (cudaStreamCreateWithFlags(&h.in, cudaStreamNonBlocking) != cudaSuccess) return SA_ERR_CUDA;
    }
    *out = &h;
    return SA_OK;
}

}  // namespace
}  // namespace sa

extern "C" int sparse_attn_fwd_host_workspace(const sa_shape* shape, size_t* bytes)
{
    if (!shape || !bytes) return SA_ERR_INVALID_ARG;
    const sa_shape s = *shape;
    if (s.B < 0 || s.Hq < 0 || s.Hkv < 0 || s.N < 0 || s.D <= 0) return SA_ERR_INVALID_ARG;
    *bytes = sa::host_layout(s).total;
    return SA_OK;
}

extern "C" int sparse_attn_fwd_host_async(const void* Q_host, const void* K_host, const void* V_host,
                                          const sa_block_mask* mask_host, const sa_pattern* pattern,
                                          const sa_shape* shape, float scale, void* O_host, float* LSE_host,
                                          void* workspace, size_t workspace_bytes, void* stream)
{
    if (!shape || !mask_host || !pattern) return SA_ERR_INVALID_ARG;
    const sa_shape s = *shape;
    if (s.B < 0 || s.Hq < 0 || s.Hkv < 0 || s.N < 0 || s.D <= 0) return SA_ERR_INVALID_ARG;
    if (s.B == 0 || s.Hq == 0 || s.N == 0) return SA_OK;
    if (s.Hkv <= 0 || s.Hq % s.Hkv != 0) return SA_ERR_UNSUPPORTED;
    if (mask_host->block != 64 && mask_host->block != 128) return SA_ERR_UNSUPPORTED;
    const int64_t T = (int64_t(s.N) + mask_host->block - 1) / mask_host->block;
    if (mask_host->n_q_tiles != T || mask_host->n_kv_tiles != T) return SA_ERR_MASK_MISMATCH;
    if (int rc = sa::check_host_mask(mask_host, T)) return rc;
    if (!Q_host || !K_host || !V_host || !O_host || !LSE_host || !workspace) return SA_ERR_INVALID_ARG;
    const sa::HostLayout L = sa::host_layout(s);
    if (workspace_bytes < L.total) return SA_ERR_BUFFER_TOO_SMALL;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return SA_ERR_MISALIGNED;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= sa::kMaxDevices) return SA_ERR_CUDA;
    std::lock_guard<std::mutex> lk(sa::g_host_mu[dev]);
    sa::HostStreams* hs = nullptr;
    if (int rc = sa::host_streams(dev, &hs)) return rc;
    // the status word exists before any chunk is queued (its first use waits for the device)
    int32_t* status = nullptr;
    if (int rc = sa::status_word(&status)) return rc;

    uint8_t* w = static_cast<uint8_t*>(workspace);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // everything queued before this call on the caller's stream comes first; the
    // inputs (and the mask copy) of the previous call on this device must have
    // been read by its kernels before they are overwritten, its outputs copied
    // back before the new kernels write theirs (its copies back may still be
    // running while this call's inputs come in)
    if (cudaEventRecord(hs->start, st) != cudaSuccess || cudaStreamWaitEvent(hs->in, hs->start, 0) != cudaSuccess ||
        cudaStreamWaitEvent(hs->in, hs->comp_done, 0) != cudaSuccess ||
        cudaStreamWaitEvent(hs->comp, hs->done, 0) != cudaSuccess)
        return SA_ERR_CUDA;
    // the mask's three arrays, each 256-aligned, at the start of the workspace
    // (its mask region is sized for the most tiles a shape can have)
    const size_t idx = (size_t(T) * 4 + 255) & ~size_t(255);
    const size_t full = idx + ((size_t(T) * T * 4 + 255) & ~size_t(255));
    const size_t bytes = full + size_t(T) * T;
    if (L.count + bytes > L.q) return SA_ERR_BUFFER_TOO_SMALL;  // cannot happen: T <= ceil(N / 64)
    sa_block_mask dmask = *mask_host;
    dmask.kv_count = reinterpret_cast<int32_t*>(w + L.count);
    dmask.kv_index = reinterpret_cast<int32_t*>(w + L.count + idx);
    dmask.kv_full = w + L.count + full;
    {
        // the same layout in the pinned stage, then one asynchronous copy
        if (cudaEventSynchronize(hs->staged) != cudaSuccess) return SA_ERR_CUDA;
        if (hs->stage_bytes < bytes) {
            if (hs->stage && cudaFreeHost(hs->stage) != cudaSuccess) return SA_ERR_CUDA;
            hs->stage = nullptr;
            hs->stage_bytes = 0;
            if (cudaHostAlloc(reinterpret_cast<void**>(&hs->stage), bytes, cudaHostAllocDefault) != cudaSuccess)
                return SA_ERR_CUDA;
            hs->stage_bytes = bytes;
        }
        std::memcpy(hs->stage, mask_host->kv_count, size_t(T) * 4);
        std::memcpy(hs->stage + idx, mask_host->kv_index, size_t(T) * T * 4);
        std::memcpy(hs->stage + full, mask_host->kv_full, size_t(T) * T);
        if (cudaMemcpyAsync(w + L.count, hs->stage, bytes, cudaMemcpyHostToDevice, hs->in) != cudaSuccess ||
            cudaEventRecord(hs->staged, hs->in) != cudaSuccess)
            return SA_ERR_CUDA;
    }

    const int64_t heads = int64_t(s.B) * s.Hkv;  // flattened kv heads
    const int64_t group = s.Hq / s.Hkv;
    int64_t first[sa::kHostChunks + 1];
    const int n_chunks = sa::host_chunks(heads, first);
    const size_t qh = size_t(s.N) * s.D * 2, lh = size_t(s.N) * 4;  // bytes of one head of Q (K, V, O) and LSE
    auto chunk_heads = [&](int c, int64_t& h0, int64_t& h1) {
        h0 = first[c];
        h1 = first[c + 1];
    };
    auto at = [](const void* p, size_t off) { return static_cast<const uint8_t*>(p) + off; };
    // every chunk's inputs first: the copy engine streams them back to back
    // while the host queues the kernels and the copies back
    for (int c = 0; c < n_chunks; c++) {
        int64_t h0, h1;
        chunk_heads(c, h0, h1);
        const size_t kv_off = size_t(h0) * qh, kv_len = size_t(h1 - h0) * qh;
        const size_t q_off = kv_off * group, q_len = kv_len * group;
        if (cudaMemcpyAsync(w + L.q + q_off, at(Q_host, q_off), q_len, cudaMemcpyHostToDevice, hs->in) !=
                cudaSuccess ||
            cudaMemcpyAsync(w + L.k + kv_off, at(K_host, kv_off), kv_len, cudaMemcpyHostToDevice, hs->in) !=
                cudaSuccess ||
            cudaMemcpyAsync(w + L.v + kv_off, at(V_host, kv_off), kv_len, cudaMemcpyHostToDevice, hs->in) !=
                cudaSuccess ||
            cudaEventRecord(hs->landed[c], hs->in) != cudaSuccess)
            return SA_ERR_CUDA;
    }
    for (int c = 0; c < n_chunks; c++) {
        int64_t h0, h1;
        chunk_heads(c, h0, h1);
        const size_t kv_off = size_t(h0) * qh, q_off = kv_off * group, q_len = size_t(h1 - h0) * qh * group;
        const size_t l_off = size_t(h0) * group * lh, l_len = size_t(h1 - h0) * group * lh;
        if (cudaStreamWaitEvent(hs->comp, hs->landed[c], 0) != cudaSuccess) return SA_ERR_CUDA;
        // the chunk as a batch of one: its kv heads and their query heads
        sa_shape cs = s;
        cs.B = 1;
        cs.Hkv = static_cast<int32_t>(h1 - h0);
        cs.Hq = static_cast<int32_t>((h1 - h0) * group);
        if (int rc = sparse_attn_fwd(w + L.q + q_off, w + L.k + kv_off, w + L.v + kv_off, &dmask, pattern, &cs, scale,
                                     w + L.o + q_off, reinterpret_cast<float*>(w + L.lse + l_off), hs->comp))
            return rc;
        if (cudaEventRecord(hs->computed[c], hs->comp) != cudaSuccess ||
            cudaStreamWaitEvent(hs->out, hs->computed[c], 0) != cudaSuccess ||
            cudaMemcpyAsync(static_cast<uint8_t*>(O_host) + q_off, w + L.o + q_off, q_len, cudaMemcpyDeviceToHost,
                            hs->out) != cudaSuccess ||
            cudaMemcpyAsync(reinterpret_cast<uint8_t*>(LSE_host) + l_off, w + L.lse + l_off, l_len,
                            cudaMemcpyDeviceToHost, hs->out) != cudaSuccess)
            return SA_ERR_CUDA;
    }
    // the caller's stream continues after the last copy back
    if (cudaEventRecord(hs->comp_done, hs->comp) != cudaSuccess || cudaEventRecord(hs->done, hs->out) != cudaSuccess ||
        cudaStreamWaitEvent(st, hs->done, 0) != cudaSuccess)
        return SA_ERR_CUDA;
    return SA_OK;
}

extern "C" int sparse_attn_fwd_host(const void* Q_host, const void* K_host, const void* V_host,
                                    const sa_block_mask* mask_host, const sa_pattern* pattern, const sa_shape* shape,
                                    float scale, void* O_host, float* LSE_host, void* workspace,
                                    size_t workspace_bytes, void* stream)
{
    const int rc = sparse_attn_fwd_host_async(Q_host, K_host, V_host, mask_host, pattern, shape, scale, O_host,
                                              LSE_host, workspace, workspace_bytes, stream);
    if (rc != SA_OK) return rc;
    if (!shape || shape->B == 0 || shape->Hq == 0 || shape->N == 0) return SA_OK;
    return sparse_attn_check_device(stream);
}

extern "C" int sparse_attn_check_device(void* stream)
{
    int32_t* status = nullptr;
    if (int rc = sa::status_word(&status)) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t word = 0;
    if (cudaMemcpyAsync(&word, status, sizeof word, cudaMemcpyDeviceToHost, st) != cudaSuccess) return SA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return SA_ERR_CUDA;
    if (word != 0) {
        if (cudaMemsetAsync(status, 0, sizeof(int32_t), st) != cudaSuccess) return SA_ERR_CUDA;
        if (cudaStreamSynchronize(st) != cudaSuccess) return SA_ERR_CUDA;
        return SA_ERR_DEVICE_TIMEOUT;
    }
    return SA_OK;
}

extern "C" int sparse_attn_set_debug(int32_t flags, int64_t timeout_cycles)
{
    std::lock_guard<std::mutex> lk(sa::g_mu);
    sa::g_debug_flags = flags;
    sa::g_timeout = timeout_cycles > 0 ? timeout_cycles : sa::kDefaultTimeout;
    return SA_OK;
}

extern "C" const char* sparse_attn_status_string(int status)
{
    switch (status) {
    case SA_OK: return "ok";
    case SA_ERR_INVALID_ARG: return "invalid argument";
    case SA_ERR_UNSUPPORTED: return "unsupported configuration";
    case SA_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case SA_ERR_BUFFER_TOO_SMALL: return "buffer too small";
    case SA_ERR_CUDA: return "CUDA error";
    case SA_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case SA_ERR_MASK_MISMATCH: return "block mask does not match N and block";
    case SA_ERR_SCRATCH_TOO_SMALL: return "block mask larger than the static scratch of the no-allocation entry point";
    default: return "unknown status";
    }
}

extern "C" int32_t sparse_attn_version(void) { return 300; }
