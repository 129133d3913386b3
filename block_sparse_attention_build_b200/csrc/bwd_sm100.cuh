// Backward pass of block-sparse causal attention on sm_100a: dQ, dK, dV for
// an upstream gradient dO, given Q, K, V, the forward output O and its LSE.
//
// The pages print no backward pass; what is computed is the gradient of the
// masked attention of the "Sparse-трансформеры" page (section "Как это
// выглядит в коде"): with P the softmax weights of each query over its
// allowed keys,
//   dV = Pᵀ dO,  dP = dO Vᵀ,  Δ_q = Σ_d dO[q,d] O[q,d],  dS = P ∘ (dP − Δ),
//   dQ = scale · dS K,  dK = scale · dSᵀ Q,
// summed over the query heads of a GQA group for dK and dV.  Tiles the block
// mask marks empty are skipped, as in the forward ("Sparse Attention" glossary
// page, section "Ein Muster in Einsparungen verwandeln").
//
// Kernels, in launch order on one stream:
//   bwd_items_kernel the work items (per kv tile and kv head, split when long);
//   bwd_prep_kernel  per query row: Δ from O and dO, the LSE in base 2, and a
//                    zeroed fp32 dQ accumulator row (and the zeroed sums of
//                    split kv tiles);
//   bwd_kernel       persistent, one CTA per SM, taking work items: an item
//                    walks the query tiles that attend to a kv tile (the
//                    transposed block mask) for every query head of the group,
//                    accumulating dK and dV in tensor memory and adding each
//                    step's dQ tile to the fp32 accumulator with reductions;
//   bwd_dq_kernel    dQ accumulator -> bf16 (and dK, dV of split kv tiles).
//
// bwd_kernel, 448 threads: warps 0-7 the element-wise work (two threads per
// kv row, tensor-memory lane = kv row), warps 8-11 the dQ read-out and
// reductions, warp 12 the TMA producer, warp 13 tensor memory allocation and
// the single MMA-issuing lane.  A step (one query tile of one head) runs as
// two half-steps of 64 query columns, double-buffered in tensor memory (half
// h in columns 128h .. 128h+127; dV, dK in 256 .. 256+2D), so that the tensor
// core computes one half while the element-wise warps work on the other:
//   Sᵀ = K Qᵀ, dPᵀ = V dOᵀ                 tcgen05 SS, N = 64, fp32 in tensor memory
//   Pᵀ = exp2(Sᵀ·scale·log2e − LSE₂)      masked on partial tiles
//   dSᵀ = Pᵀ ∘ (dPᵀ − Δ) · scale           both bf16 back into the Sᵀ columns of
//                                           tensor memory; dSᵀ also to shared memory
//   dV += Pᵀ dO, dK += dSᵀ Q               TS: A from tensor memory, K = 64
//   dQᵀ = Kᵀ dSᵀ                            SS, both operands MN-major, into the dPᵀ
//                columns with lanes = features; the dQ warps read it out
//                (releasing the buffer) and reduce it into global memory,
//                each warp instruction adding one query row's 32 consecutive
//                features (one 128-byte line).
// Every wait is bounded; on expiry a role sets a status bit, raises an abort
// flag and leaves its loop; the MMA lane drains its MMAs and the producer its
// copies before tensor memory is freed.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include <cstdint>

#include "sm100.cuh"

namespace sa {

constexpr int kBwdThreads = 448;
constexpr int kBwdElemThreads = 256;  // warps 0-7
constexpr int kBwdDqWarp0 = 8;        // warps 8-11
constexpr int kBwdDqThreads = 128;
constexpr int kBwdProducerWarp = 12;
constexpr int kBwdMmaWarp = 13;
constexpr int kBwdTile = 128;  // query and kv tile edge (the block mask's block)

enum : int32_t {
    ST_BWD_PRODUCER_WAIT = 1 << 8,
    ST_BWD_MMA_WAIT = 1 << 9,
    ST_BWD_ELEM_WAIT = 1 << 10,
    ST_BWD_DRAIN_WAIT = 1 << 11,
};

// One pattern of the backward: its transposed block mask (per kv tile the
// query tiles that attend to it) and the rule its partial tiles are masked
// with.  Window and area clipped to N; summary <= area.
struct BwdPattern {
    const int32_t* t_count;  // [T] query tiles listed for kv tile c
    const int32_t* t_index;  // [T * T] their indices, ascending
    const uint8_t* t_full;   // [T * T] 1 when every in-range pair of the tile is allowed
    int32_t window, sinks, stride, n_global, causal, area, summary;
};
constexpr int kBwdMaxPatterns = 8;
constexpr int kBwdMaxHeads = 256;
// The patterns of a backward launch and the pattern of each query head
// (different heads of a layer may carry different patterns: "Sparse-
// трансформеры" page, section "Комбинация — норма, а не исключение").
struct BwdHeads {
    BwdPattern pat[kBwdMaxPatterns];
    uint8_t head[kBwdMaxHeads];
};

constexpr int kBwdChunk = 32;  // shortest split length: lists longer than the split length are split

struct BwdParams {
    const int4* items;       // work items {kv tile, kv head, first step, steps}, split chunks first
    int32_t* n_items;        // [0] items per batch entry (the grid walks n_items * B); [1] next item to take
    const uint8_t* split;    // [T * Hkv] 1 when a tile's steps are spread over several items
    float* dk_acc;           // [B * Hkv * N * D] fp32 sums of split tiles
    float* dv_acc;
    const float* lse2;       // [B * Hq * N] LSE in base 2; +inf for a row without keys
    const float* delta;      // [B * Hq * N] Δ = rowsum(dO ∘ O)
    float* dq_acc;           // [B * Hq * N * D] fp32, zeroed by the prep kernel
    __nv_bfloat16* dK;       // [B * Hkv * N * D]
    __nv_bfloat16* dV;       // [B * Hkv * N * D]
    int32_t* status;
    long long timeout;       // SM cycles per bounded wait
    int32_t T, N, B, Hq, Hkv, group;
    int32_t n_sm;            // SMs of the device (the split length follows the per-SM share)
    int32_t split_short;     // test hook: split every list longer than kBwdChunk steps
    float scale_log2;        // scale * log2(e)
    float scale;
};

template <int D>
struct BwdCfg {
    static constexpr int kTileBytes = kBwdTile * D * 2;    // a Q, dO, K or V tile (bf16)
    static constexpr int kPanel = kBwdTile * 128;          // 64 columns x 128 rows, 128-byte swizzled
    static constexpr int kOffK = 0;
    static constexpr int kOffV = kOffK + kTileBytes;
    static constexpr int kOffQ = kOffV + kTileBytes;       // two buffers
    static constexpr int kOffdO = kOffQ + 2 * kTileBytes;  // two buffers
    static constexpr int kOffdS = kOffdO + 2 * kTileBytes; // dSᵀ: 128 kv rows x 128 q columns, two panels
    static constexpr int kOffBar = kOffdS + 2 * kPanel;
    static constexpr int kRing = 4;                          // item indices handed from the producer to the others
    static constexpr int kNumBars = 16 + 2 * kRing;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;  // tensor-memory base, abort flag, item ring
    static constexpr int kSmemBytes = kOffMisc + 16 + kRing * 4 + 1024;  // + slack to align the base to 1024
    // half h of a step: Sᵀ (fp32, then Pᵀ and dSᵀ bf16 pairs) in columns 128h ..
    // 128h+63, dPᵀ (fp32, then the half's dQᵀ with lanes = features) in 128h+64 .. +127
    static constexpr uint32_t kColdV = 256;
    static constexpr uint32_t kColdK = 256 + D;
    static constexpr uint32_t kTmemCols = 512;
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
    static_assert(kColdK + D <= kTmemCols, "tensor memory columns");
};

__device__ __forceinline__ void bwd_report(const BwdParams& p, volatile int* abort_flag, int32_t bit)
{
    *abort_flag = 1;
    atomicOr(p.status, bit);
}

// Bits lo..hi of a 32-bit word, clipped to [0, 31]; 0 when the range is empty.
__device__ __forceinline__ uint32_t bwd_bits(int lo, int hi)
{
    lo = max(lo, 0);
    hi = min(hi, 31);
    if (lo > hi) return 0u;
    const uint32_t upto_hi = hi == 31 ? 0xffffffffu : ((1u << (hi + 1)) - 1u);
    return upto_hi & ~((1u << lo) - 1u);
}

// Allowed pairs (q, kv) for q = qb + i, i in [0, 32), as bits: the pattern's
// rule (two-sided band, sink and global columns, global rows, stripe, stride)
// under causality (if set) and the sequence bound.
__device__ __forceinline__ uint32_t bwd_allow_word(const BwdPattern& p, int N, int qb, int kv)
{
    if (kv >= N) return 0u;
    const uint32_t in_range = bwd_bits((p.causal ? kv : 0) - qb, N - 1 - qb);  // (kv <=) q < N
    if (kv < max(p.sinks, p.n_global)) return in_range;
    if (p.summary > 0 && kv % p.area >= p.area - p.summary) return in_range;  // a summary column
    uint32_t m = 0u;
    if (p.window >= 0) m |= bwd_bits(kv - p.window - qb, kv + p.window - qb);
    if (p.n_global > 0) m |= bwd_bits(0, p.n_global - 1 - qb);
    if (p.area > 0) {
        const int a0 = (kv / p.area) * p.area;
        m |= bwd_bits(a0 - qb, a0 + p.area - 1 - qb);
    }
    if (p.stride > 0) {
        int i = (kv - qb) % p.stride;
        if (i < 0) i += p.stride;
        for (; i < 32; i += p.stride) m |= 1u << i;
    }
    return m & in_range;
}

__device__ __forceinline__ void red_add_f32(float* addr, float a)
{
    asm volatile("red.global.add.f32 [%0], %1;" ::"l"(addr), "f"(a) : "memory");
}

__device__ __forceinline__ void red_add_v4(float* addr, float4 v)
{
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
                 : "memory");
}

// One warp per query row: Δ = Σ_d dO·O (fp32 from the bf16 tensors), LSE₂ =
// LSE·log2(e) (+inf where LSE = -inf), and the row of the dQ accumulator zeroed.
// Rows of dK, dV in kv tiles whose steps were split: mode 0 zeroes their fp32
// sums (called from the prep kernel, before the main kernel), mode 1 writes
// them as bf16 (from the dQ conversion, after it).  The calling grid's CTAs
// stride over the (tile, batch, kv head) blocks, skipping tiles not split.
template <int D>
__device__ __forceinline__ void bwd_split_rows(const BwdParams& p, int mode)
{
    constexpr int U = D / 4;  // float4 per row
    const int n_blocks = p.T * p.B * p.Hkv;
    for (int blk = blockIdx.x; blk < n_blocks; blk += gridDim.x) {
        const int bh = blk % (p.B * p.Hkv);
        const int c = blk / (p.B * p.Hkv);
        const int hkv = bh % p.Hkv;
        if (!p.split[c * p.Hkv + hkv]) continue;
        const int rows = min(kBwdTile, p.N - c * kBwdTile);
        const int64_t base = (int64_t(bh) * p.N + int64_t(c) * kBwdTile) * U;
        for (int j = threadIdx.x; j < rows * U; j += blockDim.x) {
            const int64_t i = base + j;
            float4* ak = reinterpret_cast<float4*>(p.dk_acc) + i;
            float4* av = reinterpret_cast<float4*>(p.dv_acc) + i;
            if (mode == 0) {
                *ak = make_float4(0.f, 0.f, 0.f, 0.f);
                *av = make_float4(0.f, 0.f, 0.f, 0.f);
            } else {
                const float4 k = *ak, v = *av;
                reinterpret_cast<uint2*>(p.dK)[i] = make_uint2(pack_bf16x2(k.x, k.y), pack_bf16x2(k.z, k.w));
                reinterpret_cast<uint2*>(p.dV)[i] = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
            }
        }
    }
}

template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const __nv_bfloat16* __restrict__ O,
                                                       const __nv_bfloat16* __restrict__ dO,
                                                       const float* __restrict__ LSE, float* __restrict__ lse2,
                                                       float* __restrict__ delta, float* __restrict__ dq_acc,
                                                       int64_t rows, const BwdParams p)
{
    static_assert(D == 64 || D == 128, "head dimension");
    bwd_split_rows<D>(p, 0);  // the fp32 sums of split kv tiles start at zero
    constexpr int E = D / 32;  // elements per lane
    const int64_t row = int64_t(blockIdx.x) * 8 + threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    if (row >= rows) return;
    const __nv_bfloat16* o = O + row * D + lane * E;
    const __nv_bfloat16* g = dO + row * D + lane * E;
    float s = 0.f;
    if constexpr (E == 4) {
        const uint2 ov = *reinterpret_cast<const uint2*>(o);
        const uint2 gv = *reinterpret_cast<const uint2*>(g);
        const float2 o0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ov.x));
        const float2 o1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ov.y));
        const float2 g0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gv.x));
        const float2 g1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gv.y));
        s = o0.x * g0.x + o0.y * g0.y + o1.x * g1.x + o1.y * g1.y;
        *reinterpret_cast<float4*>(dq_acc + row * D + lane * E) = make_float4(0.f, 0.f, 0.f, 0.f);
    } else {
        const uint32_t ov = *reinterpret_cast<const uint32_t*>(o);
        const uint32_t gv = *reinterpret_cast<const uint32_t*>(g);
        const float2 o0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ov));
        const float2 g0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gv));
        s = o0.x * g0.x + o0.y * g0.y;
        *reinterpret_cast<float2*>(dq_acc + row * D + lane * E) = make_float2(0.f, 0.f);
    }
#pragma unroll
    for (int off = 16; off > 0; off /= 2) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) {
        delta[row] = s;
        const float L = LSE[row];
        lse2[row] = L == -INFINITY ? INFINITY : L * 1.44269504088896340736f;
    }
}

// dQ (bf16) from the fp32 accumulator, eight elements per thread and pass;
// then dK, dV of split kv tiles from their fp32 sums.
template <int D>
__global__ void __launch_bounds__(256) bwd_dq_kernel(const float* __restrict__ acc, __nv_bfloat16* __restrict__ dQ,
                                                     int64_t n8, const BwdParams p)
{
    bwd_split_rows<D>(p, 1);
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n8; i += int64_t(gridDim.x) * blockDim.x) {
        const float4 a = reinterpret_cast<const float4*>(acc)[2 * i];
        const float4 b = reinterpret_cast<const float4*>(acc)[2 * i + 1];
        uint4 v;
        v.x = pack_bf16x2(a.x, a.y);
        v.y = pack_bf16x2(a.z, a.w);
        v.z = pack_bf16x2(b.x, b.y);
        v.w = pack_bf16x2(b.z, b.w);
        reinterpret_cast<uint4*>(dQ)[i] = v;
    }
}

// Work items: for every (kv tile c, kv head) the steps of its query heads'
// lists, split into even chunks when longer than an SM's share of the whole
// backward (at least kBwdChunk steps), so that no CTA walks a long list alone
// (a sink tile is attended by every query tile).  Split chunks are
// listed first; one CTA of 1024 threads.
// Exclusive prefix sum over the 1024 threads of a block (warp shuffles, then
// the 32 warp totals); *total receives the sum.  Every thread must call it.
__device__ __forceinline__ long long block_exclusive_scan(long long v, long long* warp_sums, long long* total)
{
    const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
    long long x = v;
#pragma unroll
    for (int o = 1; o < 32; o *= 2) {
        const long long y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
        long long w = warp_sums[lane];
#pragma unroll
        for (int o = 1; o < 32; o *= 2) {
            const long long y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        warp_sums[lane] = w;  // inclusive over warps
        if (lane == 31) *total = w;
    }
    __syncthreads();
    const long long before = (warp > 0 ? warp_sums[warp - 1] : 0) + (x - v);
    __syncthreads();  // warp_sums may be reused by the next call
    return before;
}

__global__ void __launch_bounds__(1024) bwd_items_kernel(const BwdParams p, const __grid_constant__ BwdHeads hb,
                                                         int4* __restrict__ items, int32_t* __restrict__ n_items,
                                                         uint8_t* __restrict__ split, int32_t* __restrict__ steps_of)
{
    __shared__ long long s_warp[32];
    __shared__ long long s_total;
    const int n = p.T * p.Hkv;
    const int per = (n + 1023) / 1024;
    const int lo = min(n, static_cast<int>(threadIdx.x) * per), hi = min(n, lo + per);
    long long my_steps = 0;
    for (int idx = lo; idx < hi; idx++) {
        const int c = idx / p.Hkv, hkv = idx % p.Hkv;
        int st = 0;
        for (int h = 0; h < p.group; h++)
            st += min(max(__ldg(&hb.pat[hb.head[hkv * p.group + h]].t_count[c]), 0), p.T);
        steps_of[idx] = st;
        my_steps += st;
    }
    block_exclusive_scan(my_steps, s_warp, &s_total);
    // split length: an SM's share of all steps (every batch entry), at least kBwdChunk
    const long long share = (s_total * p.B + p.n_sm - 1) / p.n_sm;
    const int len_max =
        p.split_short ? kBwdChunk : static_cast<int>(max(static_cast<long long>(kBwdChunk), min(share, 1LL << 30)));
    int ns = 0, nu = 0;
    for (int idx = lo; idx < hi; idx++) {
        const int st = steps_of[idx];
        const int ch = st > len_max ? (st + len_max - 1) / len_max : 1;
        split[idx] = ch > 1 ? 1 : 0;
        if (ch > 1)
            ns += ch;
        else
            nu += 1;
    }
    // split chunks first, then the other tiles
    int off_s = static_cast<int>(block_exclusive_scan(ns, s_warp, &s_total));
    const int total_split = static_cast<int>(s_total);
    int off_u = total_split + static_cast<int>(block_exclusive_scan(nu, s_warp, &s_total));
    if (threadIdx.x == 0) {
        n_items[0] = total_split + static_cast<int>(s_total);
        n_items[1] = 0;  // the main kernel's CTAs take items from here
    }
    for (int idx = lo; idx < hi; idx++) {
        const int c = idx / p.Hkv, hkv = idx % p.Hkv;
        const int st = steps_of[idx];
        if (split[idx]) {
            const int ch = (st + len_max - 1) / len_max;
            const int len = (st + ch - 1) / ch;
            for (int j = 0; j < ch; j++) items[off_s++] = make_int4(c, hkv, j * len, min(len, st - j * len));
        } else {
            items[off_u++] = make_int4(c, hkv, 0, st);
        }
    }
}

// Persistent: one CTA per SM; each CTA starts with item g = blockIdx.x and
// then takes the next untaken item from a global counter (item g / B of batch
// entry g % B), so that CTAs finish together.  Its producer lane takes the
// items and hands their indices to the other roles through a small ring.  Barrier phases count steps and
// halves across items; K and V are reloaded per item once the previous item's
// MMAs are done (kv_empty), and dK, dV of tensor memory are reset per item once
// the element-wise warps have read the previous item's (acc_empty).
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmdO,
               const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, const BwdParams p,
               const __grid_constant__ BwdHeads hb)
{
    using C = BwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sK = smem + C::kOffK;
    uint8_t* sV = smem + C::kOffV;
    uint8_t* sQ = smem + C::kOffQ;
    uint8_t* sdO = smem + C::kOffdO;
    uint8_t* sdS = smem + C::kOffdS;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* kv_full = bars;        // K and V of an item landed
    uint64_t* qd_full = bars + 1;    // [2] Q and dO of a step landed
    uint64_t* qd_empty = bars + 3;   // [2] both halves' dV and dK MMAs are done with them
    uint64_t* s_full = bars + 5;     // [2] per half: Sᵀ and dPᵀ are in tensor memory
    uint64_t* ds_full = bars + 7;    // [2] per half: Pᵀ, dSᵀ written (256 element-wise threads)
    uint64_t* dq_full = bars + 9;    // [2] per half: dQᵀ in tensor memory (and every earlier MMA done)
    uint64_t* dq_empty = bars + 11;  // [2] per half: dQᵀ read out of tensor memory (128 dQ threads)
    uint64_t* drain = bars + 13;
    uint64_t* kv_empty = bars + 14;  // an item's MMAs are done with K and V
    uint64_t* acc_empty = bars + 15; // an item's dK, dV have been read out of tensor memory (256 threads)
    uint64_t* item_full = bars + 16;          // [kRing] an item index is in the ring
    uint64_t* item_empty = item_full + C::kRing;  // [kRing] every consuming warp has read it
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
    volatile int* ring = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 16);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int n_total = __ldg(p.n_items) * p.B;
    if (static_cast<int>(blockIdx.x) >= n_total) return;  // more CTAs than items (whole CTA, before any setup)
    // consumers of the item ring: the MMA warp, 8 element-wise and 4 dQ warps (one arrival each)
    constexpr int kRingReaders = 1 + kBwdElemThreads / 32 + kBwdDqThreads / 32;

    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        for (int x = 0; x < 2; x++) {
            mbar_init(&qd_full[x], 1);
            mbar_init(&qd_empty[x], 1);
            mbar_init(&s_full[x], 1);
            mbar_init(&ds_full[x], kBwdElemThreads);
            mbar_init(&dq_full[x], 1);
            mbar_init(&dq_empty[x], kBwdDqThreads);
        }
        mbar_init(drain, 1);
        mbar_init(kv_empty, 1);
        mbar_init(acc_empty, kBwdElemThreads);
        for (int i = 0; i < C::kRing; i++) {
            mbar_init(&item_full[i], 1);
            mbar_init(&item_empty[i], kRingReaders);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kBwdMmaWarp) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    if (warp == kBwdProducerWarp && lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmdO);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const long long lim = p.timeout;

    struct Item {
        int c, hkv, b, first, n;
    };
    // The k-th item of this CTA, read from the ring by a consuming warp (whole
    // warp): the global index, or n_total when the items are exhausted or a
    // wait gave up (ok cleared).
    auto next_item = [&](int k, bool& ok) -> int {
        const int slot = k % C::kRing;
        ok = __all_sync(0xffffffffu, mbar_wait(&item_full[slot], (k / C::kRing) & 1, lim));
        const int g = ok ? ring[slot] : n_total;
        __syncwarp();
        if (lane == 0) mbar_arrive(&item_empty[slot]);
        return g;
    };
    auto item_of = [&](int g) {
        const int4 it = __ldg(&p.items[g / p.B]);
        Item w;
        w.c = min(max(it.x, 0), p.T - 1);
        w.hkv = min(max(it.y, 0), p.Hkv - 1);
        w.first = max(it.z, 0);
        w.n = max(it.w, 0);
        w.b = g % p.B;
        return w;
    };
    auto list_len = [&](const Item& w, int h) {
        const BwdPattern& bp = hb.pat[hb.head[w.hkv * p.group + h]];
        return min(max(__ldg(&bp.t_count[w.c]), 0), p.T);
    };
    // query head, query tile and pattern of step j of the item's (kv tile, kv head)
    // sequence (heads outer, list entries inner)
    auto step_of = [&](const Item& w, int j, int& hq, int& r, bool& full) -> const BwdPattern& {
        int h = 0, e = j;
        for (; h < p.group - 1; h++) {
            const int n_h = list_len(w, h);
            if (e < n_h) break;
            e -= n_h;
        }
        hq = w.hkv * p.group + h;
        const BwdPattern& bp = hb.pat[hb.head[hq]];
        e = min(e, p.T - 1);
        r = min(max(__ldg(&bp.t_index[int64_t(w.c) * p.T + e]), 0), p.T - 1);
        full = __ldg(&bp.t_full[int64_t(w.c) * p.T + e]) != 0;
        return bp;
    };

    if (warp == kBwdProducerWarp) {
        // ================================================================ producer (one lane)
        if (lane == 0) {
            const uint64_t pol = policy_evict_last();
            int ia = 0;        // items with steps so far (phases of kv_full / kv_empty)
            int kq = 0;        // steps issued (Q, dO buffers)
            bool ok = true;
            for (int k = 0; ok; k++) {
                // take the next item (dynamically, so that CTAs finish together) and
                // publish its index; an index past the end ends every role's loop
                const int slot = k % C::kRing;
                if (k >= C::kRing && !mbar_wait(&item_empty[slot], ((k / C::kRing) - 1) & 1, lim)) {
                    ok = false;
                    break;
                }
                const int g = k == 0 ? static_cast<int>(blockIdx.x) : gridDim.x + atomicAdd(p.n_items + 1, 1);
                ring[slot] = min(g, n_total);
                mbar_arrive(&item_full[slot]);
                if (g >= n_total) break;
                const Item w = item_of(g);
                if (w.n == 0) continue;
                // into L2 now; the copy into shared memory waits for the previous item's MMAs
                for (int pc = 0; pc < D / 64; pc++) {
                    tma_prefetch_l2_3d(&tmK, pc * 64, w.c * kBwdTile, w.b * p.Hkv + w.hkv);
                    tma_prefetch_l2_3d(&tmV, pc * 64, w.c * kBwdTile, w.b * p.Hkv + w.hkv);
                }
                if (ia >= 1 && !mbar_wait(kv_empty, (ia - 1) & 1, lim)) {
                    ok = false;
                    break;
                }
                const int kvplane = w.b * p.Hkv + w.hkv;
                mbar_arrive_expect_tx(kv_full, 2 * C::kTileBytes);
                for (int pc = 0; pc < D / 64; pc++) {
                    tma_load_3d(sK + pc * C::kPanel, &tmK, kv_full, pc * 64, w.c * kBwdTile, kvplane, pol);
                    tma_load_3d(sV + pc * C::kPanel, &tmV, kv_full, pc * 64, w.c * kBwdTile, kvplane, pol);
                }
                ia++;
                for (int jj = 0; jj < w.n; jj++) {
                    const int buf = kq & 1;
                    if (kq >= 2 && !mbar_wait(&qd_empty[buf], ((kq >> 1) - 1) & 1, lim)) {
                        ok = false;
                        break;
                    }
                    if (*abort_flag) {
                        ok = false;
                        break;
                    }
                    int hq, r;
                    bool full;
                    step_of(w, w.first + jj, hq, r, full);
                    const int qplane = w.b * p.Hq + hq;
                    mbar_arrive_expect_tx(&qd_full[buf], 2 * C::kTileBytes);
                    for (int pc = 0; pc < D / 64; pc++) {
                        tma_load_3d(sQ + buf * C::kTileBytes + pc * C::kPanel, &tmQ, &qd_full[buf], pc * 64,
                                    r * kBwdTile, qplane, pol);
                        tma_load_3d(sdO + buf * C::kTileBytes + pc * C::kPanel, &tmdO, &qd_full[buf], pc * 64,
                                    r * kBwdTile, qplane, pol);
                    }
                    kq++;
                }
            }
            if (!ok) bwd_report(p, abort_flag, ST_BWD_PRODUCER_WAIT);
            // copies in flight land before the CTA's shared memory goes away
            bool dr = ia == 0 || mbar_wait(kv_full, (ia - 1) & 1, lim);
            for (int j = kq > 2 ? kq - 2 : 0; j < kq; j++) dr &= mbar_wait(&qd_full[j & 1], (j >> 1) & 1, lim);
            if (!dr) bwd_report(p, abort_flag, ST_BWD_DRAIN_WAIT);
        }
    } else if (warp == kBwdMmaWarp) {
        // ================================================================ MMA issuer
        // The warp runs converged; one elected lane issues each MMA and commit.
        // Within an item: Sᵀ, dPᵀ of half k + 1 (into buffer (k + 1) % 2, free
        // once the dQ warps have read the dQᵀ of the half before), then dV, dK
        // and dQᵀ of half k (once the element-wise warps have written its Pᵀ
        // and dSᵀ): the tensor core computes one half while the element-wise
        // warps work on the other.
        constexpr uint32_t id_s = idesc_bf16_f32(kBwdTile, 64, false, false);    // Sᵀ, dPᵀ: N = 64 query rows
        constexpr uint32_t id_kv = idesc_bf16_f32(kBwdTile, D, false, true);     // dV, dK
        // dQᵀ = Kᵀ dSᵀ: M = 128 feature rows (at D = 64 the upper 64 read the V
        // tile and are never used), N = 64 query rows, both operands MN-major
        constexpr uint32_t id_q = idesc_bf16_f32(kBwdTile, 64, true, true);
        constexpr uint32_t kTileU = C::kTileBytes >> 4;   // descriptor units (16 bytes)
        constexpr uint32_t kHalfRowsU = (64 * 128) >> 4;  // 64 rows of a 128-byte panel
        const uint64_t d0 = smem_desc_sw128(smem_addr(sK), 16, 1024);
        const uint32_t hi = static_cast<uint32_t>(d0 >> 32);
        const uint32_t k_km = static_cast<uint32_t>(d0);
        const uint32_t k_mn = static_cast<uint32_t>(smem_desc_sw128(smem_addr(sK), C::kPanel, 1024));
        const uint32_t v_km = static_cast<uint32_t>(smem_desc_sw128(smem_addr(sV), 16, 1024));
        const uint32_t q_km = static_cast<uint32_t>(smem_desc_sw128(smem_addr(sQ), 16, 1024));
        const uint32_t q_mn = static_cast<uint32_t>(smem_desc_sw128(smem_addr(sQ), C::kPanel, 1024));
        const uint32_t o_km = static_cast<uint32_t>(smem_desc_sw128(smem_addr(sdO), 16, 1024));
        const uint32_t o_mn = static_cast<uint32_t>(smem_desc_sw128(smem_addr(sdO), C::kPanel, 1024));
        const uint32_t s_mn = static_cast<uint32_t>(smem_desc_sw128(smem_addr(sdS), C::kPanel, 1024));
        // k-step offsets (16 elements of the contraction), in descriptor units
        auto km = [](int kk) { return static_cast<uint32_t>(((kk / 4) * C::kPanel + (kk % 4) * 32) >> 4); };
        auto mn = [](int kk) { return static_cast<uint32_t>((kk * 16 * 128) >> 4); };
        auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, lim));
        };
        auto commit = [&](uint64_t* bar) {
            if (elect_one()) tc_commit(bar);
            __syncwarp();
        };
        // Sᵀ = K Qᵀ and dPᵀ = V dOᵀ of half hf of global step q (M = kv rows, N = 64 query rows, K = D)
        auto issue_sdp = [&](int q, int hf) {
            const uint32_t bo = (q & 1) * kTileU + hf * kHalfRowsU;
            const uint32_t col = tmem + hf * 128;
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < D / 16; kk++)
                    mma_ss(col, desc_from_halves(k_km + km(kk), hi), desc_from_halves(q_km + bo + km(kk), hi), id_s,
                           kk > 0 ? 1u : 0u);
            }
            __syncwarp();
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < D / 16; kk++)
                    mma_ss(col + 64, desc_from_halves(v_km + km(kk), hi), desc_from_halves(o_km + bo + km(kk), hi),
                           id_s, kk > 0 ? 1u : 0u);
            }
            __syncwarp();
            commit(&s_full[hf]);
        };
        bool ok = true;
        bool issued = false;
        int ia = 0;   // items with steps so far
        int kq0 = 0;  // global index of the item's first step
        for (int kk_item = 0; ok; kk_item++) {
            const int g = next_item(kk_item, ok);
            if (!ok || g >= n_total) break;
            const Item w = item_of(g);
            if (w.n == 0) continue;
            const int halves = 2 * w.n;
            // K, V of this item; the first half's buffer (dQᵀ of global half 2 kq0 - 2 read out)
            ok = wait(kv_full, ia & 1) && (kq0 == 0 || wait(&dq_empty[0], (kq0 - 1) & 1)) &&
                 wait(&qd_full[kq0 & 1], (kq0 >> 1) & 1);
            if (!ok || __any_sync(0xffffffffu, *abort_flag != 0)) break;
            tc_fence_after_sync();
            issue_sdp(kq0, 0);
            issued = true;
            for (int k = 0; k < halves && ok; k++) {
                const int hf = k & 1;
                const int q = kq0 + (k >> 1);  // global step of half k
                const int kn = k + 1;
                if (kn < halves) {
                    const int qn = kq0 + (kn >> 1);
                    const int hn = 2 * kq0 + kn;  // global half index of kn
                    ok = (hn < 2 || wait(&dq_empty[hn & 1], ((hn - 2) >> 1) & 1)) &&
                         ((kn & 1) || wait(&qd_full[qn & 1], (qn >> 1) & 1));
                    if (!ok || __any_sync(0xffffffffu, *abort_flag != 0)) break;
                    tc_fence_after_sync();
                    issue_sdp(qn, kn & 1);
                }
                ok = wait(&ds_full[hf], q & 1) && (k > 0 || ia == 0 || wait(acc_empty, (ia - 1) & 1));
                if (!ok || __any_sync(0xffffffffu, *abort_flag != 0)) break;
                tc_fence_after_sync();
                const uint32_t bo = (q & 1) * kTileU + hf * kHalfRowsU;
                const uint32_t scol = tmem + hf * 128;
                // dV += Pᵀ dO and dK += dSᵀ Q over this half's 64 query rows (K = 64): A
                // from tensor memory, query columns 32u .. 32u+31 of the half hold Pᵀ
                // in packed columns 32u .. 32u+15 and dSᵀ in 32u+16 .. 32u+31
                if (elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < 4; kk++)
                        mma_ts(tmem + C::kColdV, scol + (kk / 2) * 32 + (kk % 2) * 8,
                               desc_from_halves(o_mn + bo + mn(kk), hi), id_kv, (k > 0 || kk > 0) ? 1u : 0u);
                }
                __syncwarp();
                if (elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < 4; kk++)
                        mma_ts(tmem + C::kColdK, scol + (kk / 2) * 32 + 16 + (kk % 2) * 8,
                               desc_from_halves(q_mn + bo + mn(kk), hi), id_kv, (k > 0 || kk > 0) ? 1u : 0u);
                }
                __syncwarp();
                if (hf) commit(&qd_empty[q & 1]);
                // dQᵀ = Kᵀ dSᵀ (M = feature rows, N = 64 query rows, K = kv rows), into
                // the half's dPᵀ columns; dSᵀ of half hf is panel hf of the shared tile
                if (elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < kBwdTile / 16; kk++)
                        mma_ss(scol + 64, desc_from_halves(k_mn + mn(kk), hi),
                               desc_from_halves(s_mn + hf * (C::kPanel >> 4) + mn(kk), hi), id_q, kk > 0 ? 1u : 0u);
                }
                __syncwarp();
                commit(&dq_full[hf]);
            }
            commit(kv_empty);  // every MMA of this item issued: K, V free once they complete
            kq0 += w.n;
            ia++;
        }
        if (!ok && lane == 0) bwd_report(p, abort_flag, ST_BWD_MMA_WAIT);
        // every MMA issued so far is complete before tensor memory is freed
        if (issued) {
            commit(drain);
            if (!wait(drain, 0) && lane == 0) bwd_report(p, abort_flag, ST_BWD_DRAIN_WAIT);
        }
    } else if (warp >= kBwdDqWarp0) {
        // ================================================================ dQ warps 8-11
        // Warp w reads lanes 32 (w % 4) .. +31 of each half's dQᵀ (lane = feature
        // d, columns = the half's 64 query rows), releases the columns, then adds
        // them to the fp32 accumulator: each reduction instruction covers one
        // query row's 32 consecutive features (one 128-byte line).
        const int quarter = warp % 4;
        const uint32_t lanes = static_cast<uint32_t>(quarter * 32) << 16;
        const int dcol = quarter * 32 + lane;
        bool ok = true;
        int kq0 = 0;
        for (int kk_item = 0; ok; kk_item++) {
            const int g = next_item(kk_item, ok);
            if (!ok || g >= n_total) break;
            const Item w = item_of(g);
            for (int k = 0; k < 2 * w.n; k++) {
                const int hf = k & 1;
                const int q = kq0 + (k >> 1);
                int hq, r;
                bool full;
                step_of(w, w.first + (k >> 1), hq, r, full);
                const int qh = r * kBwdTile + hf * 64;  // first query row of the half
                const int64_t qrow0 = (int64_t(w.b) * p.Hq + hq) * p.N;
                ok = __all_sync(0xffffffffu, mbar_wait(&dq_full[hf], q & 1, lim) && !*abort_flag);
                if (!ok) break;
                tc_fence_after_sync();
                uint32_t g2[64];
                tmem_ld_32x32b_x32(tmem + lanes + hf * 128 + 64, *reinterpret_cast<uint32_t(*)[32]>(&g2[0]));
                tmem_ld_32x32b_x32(tmem + lanes + hf * 128 + 96, *reinterpret_cast<uint32_t(*)[32]>(&g2[32]));
                tmem_wait_ld();
                reg_fence(*reinterpret_cast<uint32_t(*)[32]>(&g2[0]));
                reg_fence(*reinterpret_cast<uint32_t(*)[32]>(&g2[32]));
                tc_fence_before_sync();
                mbar_arrive(&dq_empty[hf]);
                if (dcol < D) {  // warp-uniform: at D = 64 quarters 2, 3 hold no feature
                    float* dst = p.dq_acc + (qrow0 + qh) * D + dcol;
                    const int nq = min(64, p.N - qh);
#pragma unroll
                    for (int i = 0; i < 64; i++)
                        if (i < nq) red_add_f32(dst + int64_t(i) * D, __uint_as_float(g2[i]));
                }
            }
            kq0 += w.n;
        }
        if (!ok && lane == 0) bwd_report(p, abort_flag, ST_BWD_ELEM_WAIT);
    } else {
        // ================================================================ element-wise warps 0-7
        // Warp w serves tensor-memory lanes 32 (w % 4) .. +31 (kv rows of Sᵀ,
        // dPᵀ, dK, dV) and, in every half, query columns 32 (w / 4) .. +31 of it.
        // Each warp decides to leave its loop as a whole (every test goes through
        // a vote); warps never wait on one another except through bounded
        // mbarrier waits.
        const int quarter = warp % 4;
        const int sub = warp / 4;
        const int t = quarter * 32 + lane;  // kv row of this thread within the tile
        const uint32_t lanes = static_cast<uint32_t>(quarter * 32) << 16;
        constexpr int kHalfD = D / 2;
        bool ok = true;
        int kq0 = 0;
        for (int kk_item = 0; ok; kk_item++) {
            const int g = next_item(kk_item, ok);
            if (!ok || g >= n_total) break;
            const Item w = item_of(g);
            const int kv = w.c * kBwdTile + t;
            const bool kv_ragged = (w.c + 1) * kBwdTile > p.N;
            for (int k = 0; k < 2 * w.n; k++) {
                const int hf = k & 1;
                const int q = kq0 + (k >> 1);
                int hq, r;
                bool full;
                const BwdPattern& bp = step_of(w, w.first + (k >> 1), hq, r, full);
                const int q0 = r * kBwdTile;
                const int qc = q0 + hf * 64 + sub * 32;  // first query column of this thread's chunk
                const int64_t qrow0 = (int64_t(w.b) * p.Hq + hq) * p.N;
                // LSE₂ and Δ of query column qc + lane, handed to the other lanes by shuffles
                const float lse_c = qc + lane < p.N ? __ldg(&p.lse2[qrow0 + qc + lane]) : INFINITY;
                const float dl_c = qc + lane < p.N ? __ldg(&p.delta[qrow0 + qc + lane]) : 0.f;
                const bool masked = !full || kv_ragged || q0 + kBwdTile > p.N;
                const uint32_t allow = masked ? bwd_allow_word(bp, p.N, qc, kv) : 0xffffffffu;
                ok = __all_sync(0xffffffffu, mbar_wait(&s_full[hf], q & 1, lim) && !*abort_flag);
                if (!ok) break;
                tc_fence_after_sync();
                const uint32_t col = hf * 128 + sub * 32;  // this chunk's Sᵀ columns; dPᵀ at +64
                uint32_t s[32], d[32];
                tmem_ld_32x32b_x32(tmem + lanes + col, s);
                tmem_ld_32x32b_x32(tmem + lanes + col + 64, d);
                tmem_wait_ld();
                reg_fence(s);
                reg_fence(d);
                uint32_t pk[16], gk[16];
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    const float l0 = __shfl_sync(0xffffffffu, lse_c, i);
                    const float l1 = __shfl_sync(0xffffffffu, lse_c, i + 1);
                    const float e0 = __shfl_sync(0xffffffffu, dl_c, i);
                    const float e1 = __shfl_sync(0xffffffffu, dl_c, i + 1);
                    float p0 = ex2_approx(fmaf(__uint_as_float(s[i]), p.scale_log2, -l0));
                    float p1 = ex2_approx(fmaf(__uint_as_float(s[i + 1]), p.scale_log2, -l1));
                    p0 = (allow >> i) & 1u ? p0 : 0.f;
                    p1 = (allow >> (i + 1)) & 1u ? p1 : 0.f;
                    const float g0 = p0 * (__uint_as_float(d[i]) - e0) * p.scale;
                    const float g1 = p1 * (__uint_as_float(d[i + 1]) - e1) * p.scale;
                    pk[i / 2] = pack_bf16x2(p0, p1);
                    gk[i / 2] = pack_bf16x2(g0, g1);
                }
                // Pᵀ and dSᵀ (bf16 pairs) over the 32 Sᵀ columns just read by this
                // thread: Pᵀ in col .. col+15, dSᵀ in col+16 .. col+31
                tmem_st_32x32b_x16(tmem + lanes + col, pk);
                tmem_st_32x32b_x16(tmem + lanes + col + 16, gk);
                // dSᵀ row t, query columns 32 sub .. +31 of the half: panel hf of the shared tile
                uint8_t* rowp = sdS + hf * C::kPanel + t * 128;
#pragma unroll
                for (int k4 = 0; k4 < 4; k4++) {
                    const int u = sub * 4 + k4;
                    *reinterpret_cast<uint4*>(rowp + ((u ^ (t & 7)) << 4)) =
                        make_uint4(gk[4 * k4], gk[4 * k4 + 1], gk[4 * k4 + 2], gk[4 * k4 + 3]);
                }
                tmem_wait_st();
                fence_proxy_async_smem();
                tc_fence_before_sync();
                mbar_arrive(&ds_full[hf]);
            }
            if (!ok) break;
            // dK and dV rows of this item, this warp's column half, after its last
            // half's MMAs (that half's dq_full): bf16 rows when the tile is one
            // item, else added to the fp32 sums (zeros when no query attends)
            const bool is_split = __ldg(&p.split[w.c * p.Hkv + w.hkv]) != 0;
            if (w.n > 0) {
                const int ql = kq0 + w.n - 1;
                ok = __all_sync(0xffffffffu, mbar_wait(&dq_full[1], ql & 1, lim) && !*abort_flag);
                if (!ok) break;
                tc_fence_after_sync();
            }
            const int64_t orow = (int64_t(w.b) * p.Hkv + w.hkv) * p.N + kv;
            // A split tile's sums go through the bytes of the dSᵀ tile that only
            // this warp writes (its rows, 16-byte units (4 sub + k) ^ (row & 7), k < 4,
            // in both panels; free once the item's last dQᵀ MMA is done): after
            // the exchange each reduction instruction adds 4 rows x 128 bytes.
            auto stage_at = [&](int r, int u) {  // row r of the warp's 32, logical 16-byte unit u < 8
                return sdS + (u >> 2) * C::kPanel + (quarter * 32 + r) * 128 + (((4 * sub + (u & 3)) ^ (r & 7)) << 4);
            };
            const int64_t row0 = (int64_t(w.b) * p.Hkv + w.hkv) * p.N + w.c * kBwdTile + quarter * 32;
#pragma unroll 1
            for (int which = 0; which < 2; which++) {
                const uint32_t col = (which == 0 ? C::kColdV : C::kColdK) + sub * kHalfD;
#pragma unroll 1
                for (int k2 = 0; k2 < kHalfD / 32; k2++) {
                    uint32_t gg[32];
                    if (w.n > 0) {
                        tmem_ld_32x32b_x32(tmem + lanes + col + k2 * 32, gg);
                        tmem_wait_ld();
                        reg_fence(gg);
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; i++) gg[i] = 0u;
                    }
                    if (is_split) {  // warp-uniform
                        __syncwarp();
#pragma unroll
                        for (int u = 0; u < 8; u++)
                            *reinterpret_cast<uint4*>(stage_at(lane, u)) =
                                make_uint4(gg[4 * u], gg[4 * u + 1], gg[4 * u + 2], gg[4 * u + 3]);
                        __syncwarp();
                        float* acc = which == 0 ? p.dv_acc : p.dk_acc;
#pragma unroll
                        for (int i = 0; i < 8; i++) {
                            const int rr = 4 * i + lane / 8;  // row within the warp's 32
                            const int u = lane % 8;
                            const float4 v = *reinterpret_cast<const float4*>(stage_at(rr, u));
                            if (w.c * kBwdTile + quarter * 32 + rr < p.N)
                                red_add_v4(acc + (row0 + rr) * D + sub * kHalfD + k2 * 32 + 4 * u, v);
                        }
                    } else if (kv < p.N) {
                        {
                            uint4* dst = reinterpret_cast<uint4*>((which == 0 ? p.dV : p.dK) + orow * D + sub * kHalfD);
#pragma unroll
                            for (int i = 0; i < 32; i += 8)
                                dst[(k2 * 32 + i) / 8] = make_uint4(
                                    pack_bf16x2(__uint_as_float(gg[i]), __uint_as_float(gg[i + 1])),
                                    pack_bf16x2(__uint_as_float(gg[i + 2]), __uint_as_float(gg[i + 3])),
                                    pack_bf16x2(__uint_as_float(gg[i + 4]), __uint_as_float(gg[i + 5])),
                                    pack_bf16x2(__uint_as_float(gg[i + 6]), __uint_as_float(gg[i + 7])));
                        }
                    }
                }
            }
            if (w.n > 0) {
                tc_fence_before_sync();
                mbar_arrive(acc_empty);  // dK, dV of tensor memory may be reset by the next item
            }
            kq0 += w.n;
        }
        if (!ok && lane == 0) bwd_report(p, abort_flag, ST_BWD_ELEM_WAIT);
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == kBwdMmaWarp) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

}  // namespace sa
