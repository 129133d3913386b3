// C ABI of the backward pass (one pattern, or a pattern per query head):
// argument checks, the workspace layout, the pattern table, TMA descriptors
// and the three launches (prep, main, dQ conversion).
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "../../include/sparse_attn.h"
#include "bwd_sm100.cuh"
#include "runtime.h"
#include "tma_host.h"

namespace sa {
namespace {

constexpr int kMaxDev = 64;
constexpr int32_t kDebugBwdSplitShort = 4;  // sparse_attn_set_debug bit 2

struct BwdLayout {
    size_t lse2, delta, dq, dk, dv, items, n_items, split, steps, total;  // byte offsets, each 256-aligned
};

// Work items: at most one per (kv tile, kv head) plus one per kBwdChunk steps
// of its list (a list holds at most group * T steps).
size_t bwd_item_capacity(const sa_shape& s)
{
    const size_t T = (size_t(s.N) + kBwdTile - 1) / kBwdTile;
    const size_t group = s.Hkv > 0 ? size_t(s.Hq) / size_t(s.Hkv) : 0;
    return T * size_t(s.Hkv) * (1 + (group * T + kBwdChunk - 1) / kBwdChunk);
}

BwdLayout bwd_layout(const sa_shape& s)
{
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    const size_t rows = size_t(s.B) * size_t(s.Hq) * size_t(s.N);
    const size_t kvrows = size_t(s.B) * size_t(s.Hkv) * size_t(s.N);
    const size_t T = (size_t(s.N) + kBwdTile - 1) / kBwdTile;
    BwdLayout w;
    w.lse2 = 0;
    w.delta = up(rows * 4);
    w.dq = w.delta + up(rows * 4);
    w.dk = w.dq + up(rows * size_t(s.D) * 4);
    w.dv = w.dk + up(kvrows * size_t(s.D) * 4);
    w.items = w.dv + up(kvrows * size_t(s.D) * 4);
    w.n_items = w.items + up(bwd_item_capacity(s) * 16);
    w.split = w.n_items + 256;
    w.steps = w.split + up(T * size_t(s.Hkv));
    w.total = w.steps + up(T * size_t(s.Hkv) * 4);
    return w;
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <int D>
int bwd_run(const void* Q, const void* K, const void* V, const void* O, const float* LSE, const void* dO,
            const BwdHeads& hb, int32_t T, const sa_shape& s, float scale, void* dQ, void* dK, void* dV, uint8_t* ws,
            cudaStream_t st)
{
    int32_t* status = nullptr;
    if (int rc = device_status_word(&status)) return rc;
    const BwdLayout L = bwd_layout(s);
    float* lse2 = reinterpret_cast<float*>(ws + L.lse2);
    float* delta = reinterpret_cast<float*>(ws + L.delta);
    float* dq_acc = reinterpret_cast<float*>(ws + L.dq);
    int4* items = reinterpret_cast<int4*>(ws + L.items);
    int32_t* n_items = reinterpret_cast<int32_t*>(ws + L.n_items);
    uint8_t* split = ws + L.split;
    int32_t* steps_scratch = reinterpret_cast<int32_t*>(ws + L.steps);
    const int64_t rows = int64_t(s.B) * s.Hq * s.N;

    CUtensorMap mq, mdo, mk, mv;
    if (!make_map_bf16_3d(&mq, Q, D, s.N, uint64_t(s.B) * s.Hq, kBwdTile) ||
        !make_map_bf16_3d(&mdo, dO, D, s.N, uint64_t(s.B) * s.Hq, kBwdTile) ||
        !make_map_bf16_3d(&mk, K, D, s.N, uint64_t(s.B) * s.Hkv, kBwdTile) ||
        !make_map_bf16_3d(&mv, V, D, s.N, uint64_t(s.B) * s.Hkv, kBwdTile))
        return SA_ERR_CUDA;

    BwdParams p;
    p.items = items;
    p.n_items = n_items;
    p.split = split;
    p.dk_acc = reinterpret_cast<float*>(ws + L.dk);
    p.dv_acc = reinterpret_cast<float*>(ws + L.dv);
    p.lse2 = lse2;
    p.delta = delta;
    p.dq_acc = dq_acc;
    p.dK = static_cast<__nv_bfloat16*>(dK);
    p.dV = static_cast<__nv_bfloat16*>(dV);
    p.status = status;
    p.timeout = wait_limit_cycles();
    p.T = T;
    p.N = s.N;
    p.B = s.B;
    p.Hq = s.Hq;
    p.Hkv = s.Hkv;
    p.group = s.Hq / s.Hkv;
    p.scale_log2 = scale * 1.44269504088896340736f;
    p.scale = scale;

    using C = BwdCfg<D>;
    static bool attr_set[kMaxDev] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return SA_ERR_CUDA;
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(bwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
            cudaSuccess)
            return SA_ERR_CUDA;
        attr_set[dev] = true;
    }
    const int n_sm = device_sm_count();
    if (n_sm <= 0) return SA_ERR_CUDA;
    p.n_sm = n_sm;
    p.split_short = (debug_flags() & kDebugBwdSplitShort) != 0;
    auto grid_for = [&](int64_t n) {
        int64_t g = (n + 255) / 256;
        if (g > int64_t(n_sm) * 8) g = int64_t(n_sm) * 8;
        return static_cast<unsigned>(g > 0 ? g : 1);
    };
    // work items; the prep kernel (row terms, zeroed dQ sums and the fp32 sums
    // of split kv tiles); the main kernel (persistent, one CTA per SM); the
    // conversions to bf16 (dQ, and dK, dV of split tiles)
    bwd_items_kernel<<<1, 1024, 0, st>>>(p, hb, items, n_items, split, steps_scratch);
    bwd_prep_kernel<D><<<static_cast<unsigned>((rows + 7) / 8), 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(O), static_cast<const __nv_bfloat16*>(dO), LSE, lse2, delta, dq_acc, rows, p);
    bwd_kernel<D><<<static_cast<unsigned>(n_sm), kBwdThreads, C::kSmemBytes, st>>>(mq, mdo, mk, mv, p, hb);
    if (cudaGetLastError() != cudaSuccess) return SA_ERR_CUDA;
    const int64_t n8 = rows * D / 8;
    bwd_dq_kernel<D><<<grid_for(n8), 256, 0, st>>>(dq_acc, static_cast<__nv_bfloat16*>(dQ), n8, p);
    return cudaGetLastError() == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

int pattern_check(const sa_pattern& pt)
{
    if (pt.window < -1 || pt.sinks < 0 || pt.stride < 0 || pt.n_global < 0 || pt.area < 0 || pt.summary < 0)
        return SA_ERR_INVALID_ARG;
    if (pt.summary > 0 && pt.area == 0) return SA_ERR_INVALID_ARG;
    if (pt.causal != 0 && pt.causal != 1) return SA_ERR_UNSUPPORTED;
    if (pt.stride > 0 && (pt.causal == 0 || pt.area > 0)) return SA_ERR_UNSUPPORTED;
    return SA_OK;
}

// The backward pass behind sparse_attn_bwd (one pattern, head_pattern null)
// and sparse_attn_bwd_heads (a pattern per query head).
int bwd_impl(const void* Q, const void* K, const void* V, const void* O, const float* LSE, const void* dO,
             const sa_block_mask* masks_t, const sa_pattern* patterns, int32_t n_patterns, const int32_t* head_pattern,
             const sa_shape* shape, float scale, void* dQ, void* dK, void* dV, void* workspace, size_t workspace_bytes,
             void* stream)
{
    if (!masks_t || !patterns || !shape) return SA_ERR_INVALID_ARG;
    const bool per_head = head_pattern != nullptr;
    if (n_patterns < 1 || n_patterns > (per_head ? kBwdMaxPatterns : 1)) return SA_ERR_INVALID_ARG;
    const sa_shape s = *shape;
    if (s.B < 0 || s.Hq < 0 || s.Hkv < 0 || s.N < 0 || s.D <= 0) return SA_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !std::isfinite(scale)) return SA_ERR_INVALID_ARG;
    for (int i = 0; i < n_patterns; i++)
        if (int rc = pattern_check(patterns[i])) return rc;
    if (s.D != 64 && s.D != 128) return SA_ERR_UNSUPPORTED;
    for (int i = 0; i < n_patterns; i++)
        if (masks_t[i].block != kBwdTile) return SA_ERR_UNSUPPORTED;
    if (s.Hq > kBwdMaxHeads) return SA_ERR_UNSUPPORTED;
    if (per_head)
        for (int h = 0; h < s.Hq; h++)
            if (head_pattern[h] < 0 || head_pattern[h] >= n_patterns) return SA_ERR_INVALID_ARG;
    if (s.B == 0 || s.Hq == 0 || s.N == 0) return SA_OK;  // nothing to compute
    if (s.Hkv <= 0 || s.Hq % s.Hkv != 0) return SA_ERR_UNSUPPORTED;
    const int64_t T = (int64_t(s.N) + kBwdTile - 1) / kBwdTile;
    for (int i = 0; i < n_patterns; i++) {
        if (masks_t[i].n_q_tiles != T || masks_t[i].n_kv_tiles != T) return SA_ERR_MASK_MISMATCH;
        if (!masks_t[i].kv_count || !masks_t[i].kv_index || !masks_t[i].kv_full) return SA_ERR_INVALID_ARG;
    }
    if (!Q || !K || !V || !O || !LSE || !dO || !dQ || !dK || !dV || !workspace) return SA_ERR_INVALID_ARG;
    if (!al16(Q) || !al16(K) || !al16(V) || !al16(O) || !al16(LSE) || !al16(dO) || !al16(dQ) || !al16(dK) ||
        !al16(dV) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return SA_ERR_MISALIGNED;
    if (workspace_bytes < bwd_layout(s).total) return SA_ERR_BUFFER_TOO_SMALL;
    const int64_t rows = int64_t(s.B) * s.Hq * s.N;
    if (int64_t(s.B) * s.Hkv * T > INT32_MAX || (rows + 7) / 8 > INT32_MAX) return SA_ERR_UNSUPPORTED;
    for (int i = 0; i < n_patterns; i++)  // the first CUDA call of the path
        if (int rc = check_device_mask(&masks_t[i])) return rc;
    BwdHeads hb{};
    for (int i = 0; i < n_patterns; i++) {
        const sa_pattern& pt = patterns[i];
        BwdPattern& bp = hb.pat[i];
        bp.t_count = masks_t[i].kv_count;
        bp.t_index = masks_t[i].kv_index;
        bp.t_full = masks_t[i].kv_full;
        bp.window = pt.window > s.N ? s.N : pt.window;  // same allowed set, no int32 overflow in the kernel
        bp.sinks = pt.sinks;
        bp.stride = pt.stride;
        bp.n_global = pt.n_global;
        bp.causal = pt.causal;
        bp.area = pt.area > s.N ? s.N : pt.area;
        bp.summary = pt.summary < pt.area ? pt.summary : pt.area;
    }
    for (int h = 0; h < s.Hq; h++) hb.head[h] = per_head ? static_cast<uint8_t>(head_pattern[h]) : 0;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const int32_t T32 = static_cast<int32_t>(T);
    if (s.D == 128) return bwd_run<128>(Q, K, V, O, LSE, dO, hb, T32, s, scale, dQ, dK, dV, ws, st);
    return bwd_run<64>(Q, K, V, O, LSE, dO, hb, T32, s, scale, dQ, dK, dV, ws, st);
}

}  // namespace
}  // namespace sa

extern "C" int sparse_attn_bwd_workspace(const sa_shape* shape, size_t* bytes)
{
    if (!shape || !bytes) return SA_ERR_INVALID_ARG;
    const sa_shape s = *shape;
    if (s.B < 0 || s.Hq < 0 || s.Hkv < 0 || s.N < 0 || s.D <= 0) return SA_ERR_INVALID_ARG;
    *bytes = sa::bwd_layout(s).total;
    return SA_OK;
}

extern "C" int sparse_attn_bwd(const void* Q, const void* K, const void* V, const void* O, const float* LSE,
                               const void* dO, const sa_block_mask* mask_t, const sa_pattern* pattern,
                               const sa_shape* shape, float scale, void* dQ, void* dK, void* dV, void* workspace,
                               size_t workspace_bytes, void* stream)
{
    return sa::bwd_impl(Q, K, V, O, LSE, dO, mask_t, pattern, 1, nullptr, shape, scale, dQ, dK, dV, workspace,
                        workspace_bytes, stream);
}

extern "C" int sparse_attn_bwd_heads(const void* Q, const void* K, const void* V, const void* O, const float* LSE,
                                     const void* dO, const sa_block_mask* masks_t, const sa_pattern* patterns,
                                     int32_t n_patterns, const int32_t* head_pattern, const sa_shape* shape,
                                     float scale, void* dQ, void* dK, void* dV, void* workspace,
                                     size_t workspace_bytes, void* stream)
{
    if (!head_pattern) return SA_ERR_INVALID_ARG;
    return sa::bwd_impl(Q, K, V, O, LSE, dO, masks_t, patterns, n_patterns, head_pattern, shape, scale, dQ, dK, dV,
                        workspace, workspace_bytes, stream);
}
