// Block-sparse causal attention forward for sm_100a.
//
// One CTA computes one 128-row query tile of one (batch, query head).  It
// walks the tile's list of live kv tiles (the compiled pattern) and never
// touches an empty tile ("Sparse Attention" glossary page, section "Ein Muster
// in Einsparungen verwandeln": speed comes from kernels that skip empty tiles).
// Per kv tile the work is the tiled exact attention of Flash-attention (the
// same page, related terms): S = Q K^T on the tensor cores, an online softmax,
// O += P V on the tensor cores.
//
// Warp roles (192 threads):
//   warp 0     TMA producer: Q once, then K and V tiles of each listed kv tile
//              into two rings of shared-memory stages
//   warp 1     allocates tensor memory; one lane issues every tcgen05.mma
//   warps 2-5  softmax: thread t owns query row t (its tensor-memory lane),
//              masks partial tiles, keeps the running max and sum, writes P
//              (bf16) into tensor memory, rescales O when the max moves far,
//              and stores O and LSE at the end
//
// Tensor memory (512 columns): S double buffer [2 x BN], O [D], P double
// buffer [2 x BN/2] (bf16 pairs).  S(j+1) = Q K(j+1)^T runs on the tensor
// cores while the softmax of tile j runs; O += P(j) V(j) follows as soon as
// P(j) is written.
//
// Every wait is bounded (`timeout` SM cycles).  On expiry the waiting role
// sets a bit in the device status word and an abort flag, everyone leaves
// their loops, in-flight copies and MMAs are waited for (again bounded), the
// tensor memory is freed and the CTA exits.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "sm100.cuh"

namespace sa {

struct FwdParams {
    const int32_t* kv_count;  // [T]
    const int32_t* kv_index;  // [T * T]
    const uint8_t* kv_full;   // [T * T]
    int32_t T;                // mask tiles per side
    int32_t N, B, Hq, Hkv, group;
    int32_t n_qtiles;         // ceil(N / 128): query tiles of 128 rows
    int32_t window, sinks, stride, n_global;
    float scale_log2;         // scale * log2(e)
    __nv_bfloat16* O;
    float* LSE;
    int32_t* status;          // device status word (bits: which wait expired)
    long long timeout;        // SM cycles per wait
    int32_t debug_flags;      // bit 0: skip the Q load (test hook)
};

enum : int32_t {
    ST_Q_WAIT = 1,
    ST_PRODUCER_WAIT = 2,
    ST_MMA_WAIT = 4,
    ST_SOFTMAX_WAIT = 8,
    ST_DRAIN_WAIT = 16,
};

constexpr int kThreads = 192;
constexpr int kBM = 128;  // query rows per CTA tile

template <int D, int BN>
struct FwdCfg {
    static constexpr int kStagesK = 2;
    static constexpr int kStagesV = 2;
    static constexpr int kQBytes = kBM * D * 2;
    static constexpr int kKVBytes = BN * D * 2;
    static constexpr int kQPanel = kBM * 128;  // 64 columns x 128 rows
    static constexpr int kKVPanel = BN * 128;  // 64 columns x BN rows
    // shared memory offsets (1024-byte aligned base)
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kQBytes;
    static constexpr int kOffV = kOffK + kStagesK * kKVBytes;
    static constexpr int kOffBar = kOffV + kStagesV * kKVBytes;
    static constexpr int kNumBars = 1 + 2 * kStagesK + 2 * kStagesV + 6 + 1;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kSmemUsed = kOffMisc + 16;
    // request at least this much so that one CTA owns the SM's tensor memory
    static constexpr int kSmemBytes = (kSmemUsed + 1024 > 120 * 1024) ? kSmemUsed + 1024 : 120 * 1024;
    // tensor memory columns
    static constexpr uint32_t kColS = 0;             // + b * BN
    static constexpr uint32_t kColO = 2 * BN;
    static constexpr uint32_t kColP = 2 * BN + D;    // + b * BN / 2
    static constexpr uint32_t kTmemCols = 512;
    static_assert(kColP + BN <= kTmemCols, "tensor memory budget");
    static_assert(kSmemUsed + 1024 <= 227 * 1024, "shared memory budget");
};

// The live kv tiles of one 128-row query tile.  With 128-wide mask tiles this
// is one row of the mask; with 64-wide tiles the query tile spans two mask
// rows and the lists are merged (a tile live in only one of them is partial
// for the whole query tile).
struct KvList {
    const int32_t* a_idx;
    const uint8_t* a_full;
    const int32_t* b_idx;
    const uint8_t* b_full;
    int a_n, b_n, pa, pb;
    bool two;

    __device__ void init(const FwdParams& p, int qtile, int BN)
    {
        const int rows_per = kBM / BN;
        const int r0 = qtile * rows_per;
        a_idx = p.kv_index + static_cast<int64_t>(r0) * p.T;
        a_full = p.kv_full + static_cast<int64_t>(r0) * p.T;
        a_n = min(max(p.kv_count[r0], 0), p.T);  // a count past the row would read the next one
        two = rows_per == 2 && r0 + 1 < p.T;
        if (two) {
            b_idx = a_idx + p.T;
            b_full = a_full + p.T;
            b_n = min(max(p.kv_count[r0 + 1], 0), p.T);
        } else {
            b_idx = nullptr;
            b_full = nullptr;
            b_n = 0;
        }
        pa = pb = 0;
    }

    __device__ bool next(int& kv, bool& full)
    {
        const bool ha = pa < a_n, hb = pb < b_n;
        if (!ha && !hb) return false;
        if (ha && hb) {
            const int x = a_idx[pa], y = b_idx[pb];
            if (x == y) {
                kv = x;
                full = a_full[pa] && b_full[pb];
                pa++;
                pb++;
            } else if (x < y) {
                kv = x;
                full = false;
                pa++;
            } else {
                kv = y;
                full = false;
                pb++;
            }
            return true;
        }
        if (ha) {
            kv = a_idx[pa];
            full = two ? false : (a_full[pa] != 0);
            pa++;
        } else {
            kv = b_idx[pb];
            full = false;
            pb++;
        }
        return true;
    }

    __device__ int count(const FwdParams& p, int qtile, int BN)
    {
        init(p, qtile, BN);
        int n = 0, kv;
        bool f;
        while (next(kv, f)) n++;
        init(p, qtile, BN);
        return n;
    }
};

__device__ __forceinline__ void report(const FwdParams& p, volatile int* abort_flag, int32_t bit)
{
    *abort_flag = 1;
    atomicOr(p.status, bit);
}

template <int D, int BN>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const FwdParams p)
{
    using C = FwdCfg<D, BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem + C::kOffQ;
    uint8_t* sK = smem + C::kOffK;
    uint8_t* sV = smem + C::kOffV;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* q_full = bars;
    uint64_t* k_full = bars + 1;
    uint64_t* k_empty = k_full + C::kStagesK;
    uint64_t* v_full = k_empty + C::kStagesK;
    uint64_t* v_empty = v_full + C::kStagesV;
    uint64_t* s_full = v_empty + C::kStagesV;  // [2]
    uint64_t* p_full = s_full + 2;             // [2]
    uint64_t* pv_done = p_full + 2;            // [2]
    uint64_t* mma_drain = pv_done + 2;         // [1]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;

    // work unit: heavier (later) query tiles first
    const int bh_count = p.B * p.Hq;
    const int qtile = p.n_qtiles - 1 - static_cast<int>(blockIdx.x) / bh_count;
    const int bh = static_cast<int>(blockIdx.x) % bh_count;
    const int b = bh / p.Hq;
    const int hq = bh % p.Hq;
    const int hkv = hq / p.group;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < C::kStagesK; s++) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
        }
        for (int s = 0; s < C::kStagesV; s++) {
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        for (int s = 0; s < 2; s++) {
            mbar_init(&s_full[s], 1);
            mbar_init(&p_full[s], 4 * 32);
            mbar_init(&pv_done[s], 1);
        }
        mbar_init(mma_drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const long long lim = p.timeout;

    KvList list;
    const int n = list.count(p, qtile, BN);

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol_q = policy_evict_first();
            const uint64_t pol_kv = policy_evict_last();
            const int q_row0 = qtile * kBM;
            const int q_plane = b * p.Hq + hq;
            const int kv_plane = b * p.Hkv + hkv;
            bool q_issued = false;
            if (n > 0 && !(p.debug_flags & 1)) {
                mbar_arrive_expect_tx(q_full, C::kQBytes);
                for (int c = 0; c < D / 64; c++)
                    tma_load_3d(sQ + c * C::kQPanel, &tmQ, q_full, c * 64, q_row0, q_plane, pol_q);
                q_issued = true;
            }
            int k_issued = 0, v_issued = 0;
            int kv;
            bool full;
            for (int j = 0; j < n && !*abort_flag; j++) {
                list.next(kv, full);
                const int sk = j % C::kStagesK, sv = j % C::kStagesV;
                if (!mbar_wait(&k_empty[sk], ((j / C::kStagesK) & 1) ^ 1, lim)) {
                    report(p, abort_flag, ST_PRODUCER_WAIT);
                    break;
                }
                mbar_arrive_expect_tx(&k_full[sk], C::kKVBytes);
                for (int c = 0; c < D / 64; c++)
                    tma_load_3d(sK + sk * C::kKVBytes + c * C::kKVPanel, &tmK, &k_full[sk], c * 64, kv * BN,
                                kv_plane, pol_kv);
                k_issued = j + 1;
                if (!mbar_wait(&v_empty[sv], ((j / C::kStagesV) & 1) ^ 1, lim)) {
                    report(p, abort_flag, ST_PRODUCER_WAIT);
                    break;
                }
                mbar_arrive_expect_tx(&v_full[sv], C::kKVBytes);
                for (int c = 0; c < D / 64; c++)
                    tma_load_3d(sV + sv * C::kKVBytes + c * C::kKVPanel, &tmV, &v_full[sv], c * 64, kv * BN,
                                kv_plane, pol_kv);
                v_issued = j + 1;
            }
            if (*abort_flag) {
                // Let copies still in flight land before the CTA's shared memory
                // goes away.  Only the newest load of each stage can be pending.
                bool ok = true;
                if (q_issued) ok &= mbar_wait(q_full, 0, lim);
                for (int t = max(0, k_issued - C::kStagesK); t < k_issued; t++)
                    ok &= mbar_wait(&k_full[t % C::kStagesK], (t / C::kStagesK) & 1, lim);
                for (int t = max(0, v_issued - C::kStagesV); t < v_issued; t++)
                    ok &= mbar_wait(&v_full[t % C::kStagesV], (t / C::kStagesV) & 1, lim);
                if (!ok) atomicOr(p.status, ST_DRAIN_WAIT);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && n > 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(kBM, BN, false, false);
            constexpr uint32_t idesc_o = idesc_bf16_f32(kBM, D, false, true);
            const uint32_t q_base = smem_addr(sQ);
            auto issue_pv = [&](int t) -> bool {
                const int pb = t & 1, sv = t % C::kStagesV;
                if (!mbar_wait(&v_full[sv], (t / C::kStagesV) & 1, lim)) return false;
                if (!mbar_wait(&p_full[pb], (t >> 1) & 1, lim)) return false;
                tc_fence_after_sync();
                const uint32_t v_base = smem_addr(sV + sv * C::kKVBytes);
#pragma unroll
                for (int kk = 0; kk < BN / 16; kk++) {
                    const uint64_t bd = smem_desc_sw128(v_base + kk * 2048, C::kKVPanel, 1024);
                    mma_ts(tmem + C::kColO, tmem + C::kColP + pb * (BN / 2) + kk * 8, bd, idesc_o,
                           (t > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(&v_empty[sv]);
                tc_commit(&pv_done[pb]);
                return true;
            };
            bool ok = mbar_wait(q_full, 0, lim);
            if (!ok) report(p, abort_flag, ST_Q_WAIT);
            for (int j = 0; ok && j < n && !*abort_flag; j++) {
                const int sb = j & 1, sk = j % C::kStagesK;
                ok = mbar_wait(&k_full[sk], (j / C::kStagesK) & 1, lim);
                if (ok && j >= 2) ok = mbar_wait(&p_full[sb], ((j - 2) >> 1) & 1, lim);  // S buffer consumed
                if (!ok) {
                    report(p, abort_flag, ST_MMA_WAIT);
                    break;
                }
                tc_fence_after_sync();
                const uint32_t k_base = smem_addr(sK + sk * C::kKVBytes);
#pragma unroll
                for (int kk = 0; kk < D / 16; kk++) {
                    const uint32_t off = (kk % 4) * 32;
                    const uint64_t ad = smem_desc_sw128(q_base + (kk / 4) * C::kQPanel + off, 16, 1024);
                    const uint64_t bd = smem_desc_sw128(k_base + (kk / 4) * C::kKVPanel + off, 16, 1024);
                    mma_ss(tmem + C::kColS + sb * BN, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
                }
                tc_commit(&k_empty[sk]);
                tc_commit(&s_full[sb]);
                if (j >= 1 && !issue_pv(j - 1)) {
                    report(p, abort_flag, ST_MMA_WAIT);
                    ok = false;
                }
            }
            if (ok && !*abort_flag && !issue_pv(n - 1)) report(p, abort_flag, ST_MMA_WAIT);
            // all issued tensor-core work finished before the memory is released
            tc_commit(mma_drain);
            if (!mbar_wait(mma_drain, 0, lim)) atomicOr(p.status, ST_DRAIN_WAIT);
        }
    } else {
        // ------------------------------------------------------------ softmax
        const int quarter = warp & 3;  // tensor-memory lanes this warp may access
        const int row = quarter * 32 + lane;
        const int q = qtile * kBM + row;
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32);
        const int cols = max(p.sinks, p.n_global);
        const bool row_all = q < p.n_global;
        float m_ref = -INFINITY;  // running max, log2 units of the scaled score
        float l_sum = 0.f;
        bool ok = true;
        int kv;
        bool full;
        for (int j = 0; j < n; j++) {
            list.next(kv, full);
            const int sb = j & 1;
            ok = mbar_wait(&s_full[sb], (j >> 1) & 1, lim);
            ok = __all_sync(0xffffffffu, ok && !*abort_flag);
            if (!ok) break;
            tc_fence_after_sync();

            float s[BN];
#pragma unroll
            for (int c = 0; c < BN; c += 32) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem_addr(tmem, lane_base, C::kColS + sb * BN + c), r);
                tmem_wait_ld();
                reg_fence(r);
#pragma unroll
                for (int i = 0; i < 32; i++) s[c + i] = __uint_as_float(r[i]);
            }

            const int kv0 = kv * BN;
            if (!full || kv0 + BN > p.N) {
                // per-element predicate, in tile-local column units
                const int dq = q - kv0;                              // causal: c <= dq
                const int c_max = min(dq, p.N - 1 - kv0);
                const int band_lo = p.window >= 0 ? dq - p.window : 1 << 30;  // band: c >= dq - window
                const int col_hi = cols - kv0;                       // columns: c < col_hi
                int next_hit = 1 << 30;                              // stride: c = dq mod s, + k s
                if (p.stride > 0) {
                    int r0 = dq % p.stride;
                    if (r0 < 0) r0 += p.stride;
                    next_hit = r0;
                }
#pragma unroll
                for (int c = 0; c < BN; c++) {
                    const bool hit = c == next_hit;
                    next_hit += hit ? p.stride : 0;
                    const bool allowed = c <= c_max && (row_all || c >= band_lo || c < col_hi || hit);
                    s[c] = allowed ? s[c] : -INFINITY;
                }
            }

            float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
            for (int c = 4; c < BN; c += 4) {
                mx0 = fmaxf(mx0, s[c]);
                mx1 = fmaxf(mx1, s[c + 1]);
                mx2 = fmaxf(mx2, s[c + 2]);
                mx3 = fmaxf(mx3, s[c + 3]);
            }
            const float m_tile = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * p.scale_log2;
            // Rescale only when the max has grown by more than 2^8: the stale
            // reference is used for O and l alike, so the result is unchanged.
            const bool grow = m_tile > m_ref + 8.f;
            float alpha = 1.f;
            if (grow) {
                alpha = ex2_approx(m_ref - m_tile);  // 0 when m_ref = -inf
                l_sum *= alpha;
                m_ref = m_tile;
            }
            const float m_use = m_ref == -INFINITY ? 0.f : m_ref;

            // P buffer sb was last read by PV(j - 2)
            if (j >= 2) {
                ok = mbar_wait(&pv_done[sb], ((j - 2) >> 1) & 1, lim);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
            }
            float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
            for (int c = 0; c < BN; c += 32) {
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; i++) {
                    const float p0 = ex2_approx(fmaf(s[c + 2 * i], p.scale_log2, -m_use));
                    const float p1 = ex2_approx(fmaf(s[c + 2 * i + 1], p.scale_log2, -m_use));
                    ls0 += p0;
                    ls1 += p1;
                    pk[i] = pack_bf16x2(p0, p1);
                }
                tmem_st_32x32b_x16(tmem_addr(tmem, lane_base, C::kColP + sb * (BN / 2) + c / 2), pk);
            }
            l_sum += ls0 + ls1;

            if (j >= 1 && __any_sync(0xffffffffu, grow)) {
                // O holds the sum up to tile j-1 once PV(j-1) is done
                ok = mbar_wait(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, lim);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                tc_fence_after_sync();
#pragma unroll
                for (int c = 0; c < D; c += 32) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(tmem_addr(tmem, lane_base, C::kColO + c), r);
                    tmem_wait_ld();
                    reg_fence(r);
#pragma unroll
                    for (int i = 0; i < 32; i++) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
                    tmem_st_32x32b_x32(tmem_addr(tmem, lane_base, C::kColO + c), r);
                }
            }
            tmem_wait_st();
            tc_fence_before_sync();
            mbar_arrive(&p_full[sb]);
        }
        if (!ok) {
            report(p, abort_flag, ST_SOFTMAX_WAIT);
        } else {
            // ------------------------------------------------------------ epilogue
            if (n > 0) {
                ok = mbar_wait(&pv_done[(n - 1) & 1], ((n - 1) >> 1) & 1, lim);
                ok = __all_sync(0xffffffffu, ok && !*abort_flag);
                if (!ok) report(p, abort_flag, ST_SOFTMAX_WAIT);
                tc_fence_after_sync();
            }
            if (ok) {
                const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
                const int64_t orow = (static_cast<int64_t>(b) * p.Hq + hq) * p.N + q;
                uint4* dst = reinterpret_cast<uint4*>(p.O + orow * D);
#pragma unroll
                for (int c = 0; c < D; c += 32) {
                    uint32_t r[32];
                    if (n > 0) {
                        tmem_ld_32x32b_x32(tmem_addr(tmem, lane_base, C::kColO + c), r);
                        tmem_wait_ld();
                        reg_fence(r);
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; i++) r[i] = 0u;
                    }
                    if (q < p.N) {
#pragma unroll
                        for (int i = 0; i < 32; i += 8) {
                            uint4 v;
                            v.x = pack_bf16x2(__uint_as_float(r[i + 0]) * inv, __uint_as_float(r[i + 1]) * inv);
                            v.y = pack_bf16x2(__uint_as_float(r[i + 2]) * inv, __uint_as_float(r[i + 3]) * inv);
                            v.z = pack_bf16x2(__uint_as_float(r[i + 4]) * inv, __uint_as_float(r[i + 5]) * inv);
                            v.w = pack_bf16x2(__uint_as_float(r[i + 6]) * inv, __uint_as_float(r[i + 7]) * inv);
                            dst[(c + i) / 8] = v;
                        }
                    }
                }
                if (q < p.N)
                    p.LSE[orow] = l_sum > 0.f ? (m_ref + log2f(l_sum)) * 0.69314718055994530942f : -INFINITY;
            }
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

}  // namespace sa
