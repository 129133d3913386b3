// sparse_attn_fwd_noalloc: the forward pass for callers that cannot allocate
// device memory.
//
// Some callers reserve all the device memory they will ever use when they
// start (a pool of their own) and must not allocate afterwards: cudaMalloc can
// block the host and stall other work on the device, and it can fail under
// memory pressure in the middle of a request.  sparse_attn_fwd allocates a
// small status word on its first call on a device and needs the block mask in
// device memory the caller allocated.  This entry point needs neither: its
// scratch (the status word and a device copy of the block mask) lives in the
// file-scope array below, which the library's module holds on every GPU that
// loads it, until the process exits.
//
// The array's name is a host-side stand-in, not a device address.  The first
// call on a device looks its device address up with cudaGetSymbolAddress, with
// that device current, and keeps it; make that first call before any stream
// capture.  All calls share the array and it keeps the last call's contents:
// the status word is cleared on every call and the mask region rewritten.
// Calls whose kernels overlap on the GPU race on it; each call waits for its
// stream before returning, and calls from several host threads are serialised
// per device here.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/sparse_attn.h"
#include "fwd_sm100.cuh"
#include "runtime.h"
#include "tma_host.h"

namespace sa {
namespace noalloc {

static __device__ __align__(256) uint8_t g_scratch[SA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
constexpr size_t kStatusBytes = 256;  // the status word, padded to keep the mask 256-byte aligned

std::mutex g_mu[kMaxDevices];
uint8_t* g_addr[kMaxDevices] = {};
bool g_attr[kMaxDevices][4] = {};

size_t align16(size_t x) { return (x + 15) & ~size_t(15); }

// Bytes of scratch a mask with T tiles per side needs.
size_t scratch_bytes(int64_t T)
{
    return kStatusBytes + align16(size_t(T) * 4) + align16(size_t(T) * size_t(T) * 4) + size_t(T) * size_t(T);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <int D, int BN>
int launch(int dev, int which, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
           const CUtensorMap& mo, const FwdParams& p, int grid, cudaStream_t stream)
{
    using C = FwdCfg<D, BN>;
    auto kern = fwd_kernel<D, BN, false>;
    if (!g_attr[dev][which]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess)
            return SA_ERR_CUDA;
        // the warpgroups' register split must fit what the kernel is launched with
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return SA_ERR_CUDA;
        if (fa.numRegs * kThreads < kRegSplitTotal) return SA_ERR_UNSUPPORTED;
        g_attr[dev][which] = true;
    }
    const HeadPatterns hp{};  // one pattern: the per-head table is not read
    kern<<<grid, kThreads, C::kSmemBytes, stream>>>(mq, mk, mv, mo, p, hp);
    return cudaGetLastError() == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

}  // namespace noalloc
}  // namespace sa

extern "C" int sparse_attn_fwd_noalloc(const void* Q, const void* K, const void* V, const sa_block_mask* mask,
                                       const sa_pattern* pattern, const sa_shape* shape, float scale, void* O,
                                       float* LSE, void* stream)
{
    using namespace sa;
    using namespace sa::noalloc;
    if (!mask || !pattern || !shape) return SA_ERR_INVALID_ARG;
    const sa_shape s = *shape;
    if (s.B < 0 || s.Hq < 0 || s.Hkv < 0 || s.N < 0 || s.D <= 0) return SA_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !std::isfinite(scale)) return SA_ERR_INVALID_ARG;
    // the causal band / sinks / stride / global forms only (no pattern table here)
    if (pattern->causal != 1 || pattern->area != 0 || pattern->summary != 0) return SA_ERR_UNSUPPORTED;
    if (pattern->window < -1 || pattern->sinks < 0 || pattern->stride < 0 || pattern->n_global < 0)
        return SA_ERR_INVALID_ARG;
    if (s.D != 64 && s.D != 128) return SA_ERR_UNSUPPORTED;
    if (mask->block != 64 && mask->block != 128) return SA_ERR_UNSUPPORTED;
    if (s.B == 0 || s.Hq == 0 || s.N == 0) return SA_OK;
    if (s.Hkv <= 0 || s.Hq % s.Hkv != 0) return SA_ERR_UNSUPPORTED;
    const int64_t T = (int64_t(s.N) + mask->block - 1) / mask->block;
    if (mask->n_q_tiles != T || mask->n_kv_tiles != T) return SA_ERR_MASK_MISMATCH;
    if (scratch_bytes(T) > SA_NOALLOC_SCRATCH_BYTES) return SA_ERR_SCRATCH_TOO_SMALL;
    if (!Q || !K || !V || !O || !LSE) return SA_ERR_INVALID_ARG;
    // the mask is read on the host: a malformed one is refused before any device work
    if (int rc = check_host_mask(mask, T)) return rc;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || (reinterpret_cast<uintptr_t>(LSE) & 3u))
        return SA_ERR_MISALIGNED;
    const int64_t n_qtiles = (int64_t(s.N) + kBM - 1) / kBM;
    const int64_t group = s.Hq / s.Hkv;
    const int64_t pairs = group >= 2 ? (group + 1) / 2 : (n_qtiles + 1) / 2;
    const int64_t n_units = group >= 2 ? n_qtiles * s.B * s.Hkv * pairs : pairs * s.B * s.Hq;
    if (n_units > INT32_MAX || int64_t(s.B) * s.Hq > INT32_MAX) return SA_ERR_UNSUPPORTED;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SA_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu[dev]);
    if (!g_addr[dev]) {
        // once per device, with this device current
        void* addr = nullptr;
        if (cudaGetSymbolAddress(&addr, g_scratch) != cudaSuccess || !addr) return SA_ERR_CUDA;
        g_addr[dev] = static_cast<uint8_t*>(addr);
    }
    int n_sm = 0;
    if (cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n_sm <= 0)
        return SA_ERR_CUDA;

    uint8_t* base = g_addr[dev];
    int32_t* status = reinterpret_cast<int32_t*>(base);
    int32_t* d_count = reinterpret_cast<int32_t*>(base + kStatusBytes);
    int32_t* d_index = reinterpret_cast<int32_t*>(base + kStatusBytes + align16(size_t(T) * 4));
    uint8_t* d_full = base + kStatusBytes + align16(size_t(T) * 4) + align16(size_t(T) * size_t(T) * 4);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(status, 0, sizeof(int32_t), st) != cudaSuccess ||
        cudaMemcpyAsync(d_count, mask->kv_count, size_t(T) * 4, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(d_index, mask->kv_index, size_t(T) * size_t(T) * 4, cudaMemcpyHostToDevice, st) !=
            cudaSuccess ||
        cudaMemcpyAsync(d_full, mask->kv_full, size_t(T) * size_t(T), cudaMemcpyHostToDevice, st) != cudaSuccess)
        return SA_ERR_CUDA;

    CUtensorMap mq, mk, mv, mo;
    const uint32_t bn = static_cast<uint32_t>(mask->block);
    if (!make_map_bf16_3d(&mq, Q, s.D, s.N, uint64_t(s.B) * s.Hq, kBM) ||
        !make_map_bf16_3d(&mk, K, s.D, s.N, uint64_t(s.B) * s.Hkv, bn) ||
        !make_map_bf16_3d(&mv, V, s.D, s.N, uint64_t(s.B) * s.Hkv, bn) ||
        !make_map_bf16_3d(&mo, O, s.D, s.N, uint64_t(s.B) * s.Hq, bn))
        return SA_ERR_CUDA;

    FwdParams p;
    p.kv_count = d_count;
    p.kv_index = d_index;
    p.kv_full = d_full;
    p.T = static_cast<int32_t>(T);
    p.N = s.N;
    p.B = s.B;
    p.Hq = s.Hq;
    p.Hkv = s.Hkv;
    p.group = static_cast<int32_t>(group);
    p.n_qtiles = static_cast<int32_t>(n_qtiles);
    p.n_units = static_cast<int32_t>(n_units);
    int64_t n_whole = 0, n_items = 0;
    plan_items(n_units, n_sm, false, &n_whole, &n_items);
    if (n_items > INT32_MAX) return SA_ERR_UNSUPPORTED;
    p.n_whole = static_cast<int32_t>(n_whole);
    p.n_items = static_cast<int32_t>(n_items);
    p.pairs = static_cast<int32_t>(pairs);
    p.window = pattern->window > s.N ? s.N : pattern->window;  // same allowed set, no int32 overflow in the kernel
    p.sinks = pattern->sinks;
    p.stride = pattern->stride;
    p.n_global = pattern->n_global;
    p.scale_log2 = scale * 1.44269504088896340736f;
    p.O = static_cast<__nv_bfloat16*>(O);
    p.LSE = LSE;
    p.status = status;
    p.timeout = wait_limit_cycles();
    p.debug_flags = debug_flags() & 1;  // the skip-Q-load test hook; work units are never split here
    p.snake = snake_order(sa_block_mask_fields{T, mask->n_live, mask->max_per_row});
    const int grid = static_cast<int>(n_items < n_sm ? n_items : n_sm);
    int rc;
    if (s.D == 128 && bn == 128)
        rc = launch<128, 128>(dev, 0, mq, mk, mv, mo, p, grid, st);
    else if (s.D == 64 && bn == 128)
        rc = launch<64, 128>(dev, 1, mq, mk, mv, mo, p, grid, st);
    else if (s.D == 128)
        rc = launch<128, 64>(dev, 2, mq, mk, mv, mo, p, grid, st);
    else
        rc = launch<64, 64>(dev, 3, mq, mk, mv, mo, p, grid, st);
    if (rc != SA_OK) return rc;

    int32_t word = 0;
    if (cudaMemcpyAsync(&word, status, sizeof word, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return SA_ERR_CUDA;
    return word != 0 ? SA_ERR_DEVICE_TIMEOUT : SA_OK;
}
