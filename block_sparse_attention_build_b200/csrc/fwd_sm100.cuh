// Block-sparse causal attention forward for sm_100a.
//
// Persistent kernel: one CTA per SM walks a strided share of the work units.
// A work unit is two 128-row query tiles ("slots" A and B) that read the same
// key/value head: two query heads of one group at the same query tile when
// heads are grouped, else two consecutive query tiles of one head.  The unit
// walks the union of the slots' lists of live kv tiles (the compiled pattern)
// and never touches a tile outside it ("Sparse Attention" glossary page,
// section "Ein Muster in Einsparungen verwandeln": speed comes from kernels
// that skip empty tiles).  Per kv tile the work is the tiled exact attention
// of Flash-attention (same page, related terms): S = Q K^T on the tensor
// cores, an online softmax, O += P V on the tensor cores.
//
// Warp roles (384 threads, three warpgroups):
//   warp 0     producer: builds each unit's step list (the union of the
//              slots' live kv tiles) into a two-entry shared-memory ring that
//              the other roles read, TMA-loads Q of both slots, and streams the
//              unit's items through one ring of shared-memory stages: K and V
//              of every step, then, per slot, the stages that will hold that
//              slot's O tile (granted without a load)
//   warp 1     allocates tensor memory; one lane issues every tcgen05.mma
//   warp 2     O store: TMA-stores each staged O tile and hands its stages
//              back to the producer once the store has read them
//   warp 3     idle
//   warps 4-7  softmax of slot A, warps 8-11 softmax of slot B: thread t of a
//              group owns query row t (its tensor-memory lane), masks partial
//              tiles, keeps the running max and sum, writes P (bf16) over its
//              S in tensor memory, rescales O when the max moves far, and at
//              the end of the unit writes its normalised O row (bf16) into the
//              granted ring stage and its LSE to global memory
// The first warpgroup gives registers up (88 per thread) so that the softmax
// warpgroups can hold a whole row of S (208 per thread): 128 x 88 + 256 x 208
// equals the 384 x 168 the block is launched with.
//
// Ping-pong: the MMA warp issues PV_A(j), S_A(j+1), PV_B(j), S_B(j+1), so the
// tensor cores work on one slot while the other slot's softmax runs.
//
// Split units: when the units do not fill the last round of CTAs evenly, the
// units of that round are split: each of their query tiles becomes a unit of
// its own whose two slots hold the same 128 rows, slot A walking the first
// half of the tile's kv list and slot B the second.  Each slot then streams
// its own K and V, and at the end slot A's threads merge the two partial
// results row by row (both accumulators live in the same tensor-memory lanes):
// with M the larger running max, O = (O_A 2^(m_A - M) + O_B 2^(m_B - M)) /
// (l_A 2^(m_A - M) + l_B 2^(m_B - M)).  The busiest CTA then does about half a
// unit more than the mean instead of a whole unit.
//
// Unit boundaries: a slot's Q buffer is handed back by a commit after the
// slot's last S MMA of the unit, so the next unit's Q is loaded while the last
// step's softmax and PV run; the O tile goes out through ring stages, so
// nothing waits for the store before the next unit's first S.
//
// Tensor memory (512 columns): S_A, S_B [BN each], O_A, O_B [D each].  P_X
// (bf16 pairs, BN/2 columns) is written over the first columns of S_X once S_X
// has been read; the next S_X MMA is issued after PV_X, and tcgen05.mma
// operations issued by one thread execute in issue order.  A commit after
// S_X(j) also covers PV_X(j-1), so when the softmax sees S_X(j), O_X holds
// every product up to tile j-1.
//
// Every wait is bounded (`timeout` SM cycles).  On expiry the waiting role sets
// a bit in the device status word and an abort flag, everyone leaves their
// loops, in-flight copies and MMAs are waited for (again bounded), the tensor
// memory is freed and the CTA exits.
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
    int32_t n_units;          // work units of two slots
    int32_t n_whole;          // units processed whole; units n_whole.. are split
    int32_t n_items;          // n_whole + 2 * (n_units - n_whole): what the CTAs walk
    int32_t pairs;            // grouped: ceil(group / 2); else ceil(n_qtiles / 2)
    int32_t window, sinks, stride, n_global;
    float scale_log2;         // scale * log2(e)
    __nv_bfloat16* O;
    float* LSE;
    int32_t* status;          // device status word (bits: which wait expired)
    long long timeout;        // SM cycles per wait
    int32_t debug_flags;      // bit 0: skip the first Q load (test hook)
    int32_t snake;            // 1: the CTAs take work items in snake order (see unit_of)
};

// Per-head patterns: each query head follows one of up to kMaxPatterns
// compiled patterns (its block mask and the rule parameters its partial tiles
// are masked with).  Different heads of a layer may carry different patterns
// ("Sparse-трансформеры" page, section "Комбинация — норма, а не
// исключение").  Used by the kernels instantiated with MULTI = true, which
// also take the pattern forms beyond causal band / sinks / stride / global:
// no causality (two-sided band) and stripes (Area Attention, "Sparse
// Attention" glossary page, section "Anwendungen").
constexpr int kMaxPatterns = 8;
constexpr int kMaxHeadsMulti = 256;
struct PatternRef {
    const int32_t* kv_count;  // [T]
    const int32_t* kv_index;  // [T * T]
    const uint8_t* kv_full;   // [T * T]
    int32_t window, sinks, stride, n_global, causal, area, summary;  // summary <= area
    // mode 1: the residual stride pass of the stride-aware path, on tokens
    // grouped by residue (position P = (t mod stride) * area + t / stride): row P
    // of group g = P / area allows the one interval [g * area + ceil((col_lo - g) /
    // stride), P - shift] (stride pairs not already in the band, the sink or
    // global columns or a global row)
    int32_t mode, shift, col_lo;
};
struct HeadPatterns {
    PatternRef pat[kMaxPatterns];
    uint8_t head[kMaxHeadsMulti];  // pattern of each query head
    // > 0: the tensor maps view the residue-grouped order P = (t mod grp_s) *
    // grp_n + t / grp_s of token-order tensors as 4-D (feature, P / grp_n,
    // P mod grp_n, plane); LSE and zeroed O rows go to token t
    int32_t grp_n, grp_s;
};

enum : int32_t {
    ST_Q_WAIT = 1,
    ST_PRODUCER_WAIT = 2,
    ST_MMA_WAIT = 4,
    ST_SOFTMAX_WAIT = 8,
    ST_DRAIN_WAIT = 16,
    ST_STORE_WAIT = 32,
};

constexpr int kThreads = 384;
constexpr int kRegsControl = 88;
constexpr int kRegsSoftmax = 208;
// Registers the split hands out; the kernel must be launched with at least this
// many (threads x registers per thread at launch), or setmaxnreg.inc would wait
// forever.  The launchers check the compiled count before the first launch.
constexpr int kRegSplitTotal = 128 * kRegsControl + 256 * kRegsSoftmax;
static_assert(kRegSplitTotal <= kThreads * 168, "register split");
constexpr int kBM = 128;  // query rows per slot
// Largest number of kv tiles per side the kernel handles (the per-unit step
// list is staged in shared memory with 14-bit tile indices).
constexpr int kMaxTiles = 4096;

// Bytes of shared memory for the ring of K / V / O stages.
constexpr int kRingBytes = 128 * 1024;

template <int D, int BN>
struct FwdCfg {
    static constexpr int kQBytes = kBM * D * 2;
    static constexpr int kKVBytes = BN * D * 2;             // one ring stage: a K or V tile, or BN rows of O
    static constexpr int kStages = kRingBytes / kKVBytes;   // 4 (D = BN = 128) to 16 (D = BN = 64)
    static constexpr int kOBlocks = kBM / BN;               // ring stages per slot's O tile
    static constexpr int kQPanel = kBM * 128;  // 64 columns x 128 rows
    static constexpr int kKVPanel = BN * 128;  // 64 columns x BN rows
    static constexpr int kOffQ = 0;            // two slots
    static constexpr int kOffRing = kOffQ + 2 * kQBytes;
    // unit-info ring: per unit its kv steps, 16 bits each (kv tile | fullA << 14 | fullB << 15)
    static constexpr int kOffList = kOffRing + kStages * kKVBytes;
    static constexpr int kOffListN = kOffList + 2 * kMaxTiles * 2;              // int[2] steps, int[2] ring positions
    static constexpr int kOffBitmap = kOffListN + 16;                          // live + 4 full bitmaps
    static constexpr int kOffBar = kOffBitmap + 5 * (kMaxTiles / 32) * 4 + 2 * kBM * 4;
    static constexpr int kOffMLX = kOffBitmap + 5 * (kMaxTiles / 32) * 4;     // [2][kBM] fp32: slot B's max, sum
    static constexpr int kNumBars = 2 * kStages + 2 * 7 + 2 * 2 + 1 + 2;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kSmemUsed = kOffMisc + 16;
    // at least this much, so that one CTA owns the SM's tensor memory
    static constexpr int kSmemBytes = (kSmemUsed + 1024 > 120 * 1024) ? kSmemUsed + 1024 : 120 * 1024;
    static constexpr uint32_t kTmemCols = 512;
    static_assert(kStages >= 4 && kRingBytes % kKVBytes == 0, "ring of at least four stages");
    static_assert(2 * BN + 2 * D <= 512, "tensor memory budget");
    static_assert(kSmemUsed + 1024 <= 227 * 1024, "shared memory budget");
};

// The scalar fields of a compiled block mask that the scheduling choice reads.
struct sa_block_mask_fields {
    int64_t T, n_live;
    int32_t max_per_row;
};

// Work items (host side).  Units that fill whole rounds of the CTAs run whole.
// When the rest would give at most half of the CTAs one more unit, those units
// are split, two items each, so that the last round costs about half a unit;
// so are all units when there are at most half as many as CTAs (a small
// problem: the idle CTAs then take half of every list).  `split_all` (a test
// switch) splits every unit.
inline void plan_items(int64_t n_units, int64_t n_ctas, bool split_all, int64_t* n_whole, int64_t* n_items)
{
    int64_t whole = n_units;
    if (split_all || 2 * n_units <= n_ctas) {
        whole = 0;
    } else if (n_units > n_ctas) {
        const int64_t r = n_units % n_ctas;
        if (r > 0 && 2 * r <= n_ctas) whole = n_units - r;
    }
    *n_whole = whole;
    *n_items = whole + 2 * (n_units - whole);
}

// Work item of this CTA in its round k.  Items are ordered heaviest first and
// CTA c takes item c of every round, or, with `snake` (rows of the mask whose
// lengths vary widely), item G - 1 - c of odd rounds (G CTAs), so that a CTA
// that drew a heavier item in one round draws a lighter one in the next.
// Every item is taken once, and a CTA's items grow with k: the first one past
// the end ends its walk.
__device__ __forceinline__ int unit_of(int k, int snake)
{
    const int G = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
    return k * G + ((snake & k & 1) ? G - 1 - c : c);
}

// Snake order when the mask's rows vary widely in length: their mean live
// tiles below 3/5 of the longest row (from the mask's scalar fields; a
// scheduling choice only, any value is safe).  Measured: the strided + global
// workload (mean / longest 0.50) 10 % faster; the windowed workloads (0.81 to
// 0.99) and Area Attention (0.67) keep the plain order, which was as fast or
// 1-1.5 % faster there.
inline int32_t snake_order(const sa_block_mask_fields& f)
{
    return (f.max_per_row > 0 && f.T > 0 && 5 * f.n_live < 3 * int64_t(f.max_per_row) * f.T) ? 1 : 0;
}

// Debug flag: split every unit (exercises the split path on small problems).
constexpr int32_t kDebugSplitAll = 2;

// One work unit: up to two slots, each a 128-row query tile of one head.
struct Unit {
    int b, hkv;
    int hq[2];
    int qtile[2];
    bool valid[2];
    bool split;  // one query tile: slot A takes the first half of its kv list, slot B the second
};

__device__ __forceinline__ Unit decode_pair(const FwdParams& p, int u)
{
    Unit w;
    w.split = false;
    if (p.group >= 2) {
        // u = ((n_qtiles - 1 - i) * B * Hkv + b * Hkv + hkv) * pairs + g: later (heavier) tiles first
        const int g = u % p.pairs;
        const int r = u / p.pairs;
        const int bh = r % (p.B * p.Hkv);
        const int i = p.n_qtiles - 1 - r / (p.B * p.Hkv);
        w.b = bh / p.Hkv;
        w.hkv = bh % p.Hkv;
        w.hq[0] = w.hkv * p.group + 2 * g;
        w.hq[1] = w.hq[0] + 1;
        w.qtile[0] = w.qtile[1] = i;
        w.valid[0] = true;
        w.valid[1] = 2 * g + 1 < p.group;
    } else {
        // u = (pairs - 1 - pp) * B * Hq + b * Hq + h; the slots are q-tiles 2 pp and 2 pp + 1
        const int bh = u % (p.B * p.Hq);
        const int pp = p.pairs - 1 - u / (p.B * p.Hq);
        w.b = bh / p.Hq;
        w.hkv = bh % p.Hq;
        w.hq[0] = w.hq[1] = w.hkv;
        w.qtile[0] = 2 * pp;
        w.qtile[1] = 2 * pp + 1;
        w.valid[0] = true;
        w.valid[1] = 2 * pp + 1 < p.n_qtiles;
    }
    return w;
}

// Work item t of the CTAs' walk: a whole unit, or one query tile of a split unit.
__device__ __forceinline__ Unit decode_unit(const FwdParams& p, int t)
{
    if (t < p.n_whole) return decode_pair(p, t);
    const int s = t - p.n_whole;
    const Unit pr = decode_pair(p, p.n_whole + s / 2);
    const bool x = s & 1;
    Unit w = pr;
    w.hq[0] = w.hq[1] = x ? pr.hq[1] : pr.hq[0];
    w.qtile[0] = w.qtile[1] = x ? pr.qtile[1] : pr.qtile[0];
    w.valid[0] = w.valid[1] = x ? pr.valid[1] : pr.valid[0];
    w.split = true;
    return w;
}

// Steps of slot x in a unit whose step list has n entries, and the list entry
// of its step j.
__device__ __forceinline__ int slot_steps(const Unit& w, int n, int x)
{
    if (!(x ? w.valid[1] : w.valid[0])) return 0;
    if (!w.split) return n;
    return x == 0 ? (n + 1) / 2 : n / 2;
}
__device__ __forceinline__ int slot_entry(const Unit& w, int n, int x, int j)
{
    return (w.split && x == 1) ? (n + 1) / 2 + j : j;
}
// Ring items of a unit, relative to its first: a whole unit loads K(j), V(j)
// per step (2n items); a split unit loads K_A(j), K_B(j), V_A(j), V_B(j) while
// both halves have a step j, then K_A(j), V_A(j) (again 2n items in all).
__device__ __forceinline__ int k_item(const Unit& w, int n, int x, int j)
{
    if (!w.split) return 2 * j;
    const int nb = n / 2;
    return j < nb ? 4 * j + x : 4 * nb + 2 * (j - nb);
}
__device__ __forceinline__ int v_item(const Unit& w, int n, int x, int j)
{
    if (!w.split) return 2 * j + 1;
    const int nb = n / 2;
    return j < nb ? 4 * j + 2 + x : 4 * nb + 2 * (j - nb) + 1;
}
// Ring stages holding O tiles at the end of a unit: one slot's for a split unit.
__device__ __forceinline__ int o_slots(const Unit& w) { return (w.split || !w.valid[1]) ? 1 : 2; }

// Bits lo..hi (inclusive) of a 32-bit word, clipped to 0..31; 0 when empty.
__device__ __forceinline__ uint32_t bits_between(int lo, int hi)
{
    lo = max(lo, 0);
    hi = min(hi, 31);
    return lo > hi ? 0u : ((0xffffffffu >> (31 - hi)) & (0xffffffffu << lo));
}

// Build the step list of work unit w (whole warp, converged): the ascending
// union of the live kv tiles of the unit's mask rows, each entry
// kv | fullA << 14 | fullB << 15, where a slot's flag is set when every
// existing mask row of that slot marks the tile full.  The rows are read with
// coalesced loads into shared-memory bitmaps (bm: live, then one full bitmap
// per row, kMaxTiles / 32 words each), then a warp prefix scan emits the set
// bits in order.  Returns the number of steps (the same in every lane).
template <bool MULTI>
__device__ __forceinline__ int build_unit_list(const FwdParams& p, const HeadPatterns& hp, const Unit& w, int BN,
                                               uint16_t* list, uint32_t* bm, int lane)
{
    // the block mask each slot's rows come from
    const int32_t* cnt_of[2];
    const int32_t* idx_of[2];
    const uint8_t* full_of[2];
#pragma unroll
    for (int x = 0; x < 2; x++) {
        if constexpr (MULTI) {
            // an absent slot B may name head Hq (one past the table): use slot A's
            const PatternRef& pr = hp.pat[hp.head[(x && w.valid[1]) ? w.hq[1] : w.hq[0]]];
            cnt_of[x] = pr.kv_count;
            idx_of[x] = pr.kv_index;
            full_of[x] = pr.kv_full;
        } else {
            cnt_of[x] = p.kv_count;
            idx_of[x] = p.kv_index;
            full_of[x] = p.kv_full;
        }
    }
    constexpr int W = kMaxTiles / 32;
    const int rows_per = kBM / BN;
    const int words = (p.T + 31) / 32;
    int row[4], cnt[4], kv0[4];
    bool exists[4], full0[4];
    // one round trip: each row's count and its first 32 entries are loaded
    // together (lane < T keeps every load inside the row)
#pragma unroll
    for (int r = 0; r < 4; r++) {
        const int x = r / 2, k = r % 2;
        row[r] = w.qtile[x] * rows_per + k;
        exists[r] = w.valid[x] && k < rows_per && row[r] < p.T;
        const int64_t off = static_cast<int64_t>(exists[r] ? row[r] : 0) * p.T + lane;
        const bool in_row = exists[r] && lane < p.T;
        cnt[r] = exists[r] ? __ldg(&cnt_of[x][row[r]]) : 0;
        kv0[r] = in_row ? __ldg(&idx_of[x][off]) : -1;
        full0[r] = in_row ? __ldg(&full_of[x][off]) != 0 : false;
    }
#pragma unroll
    for (int r = 0; r < 4; r++) cnt[r] = min(max(cnt[r], 0), p.T);  // clamp a corrupt count: never read past the row
    for (int i = lane; i < words; i += 32) {
        bm[i] = 0u;
#pragma unroll
        for (int r = 0; r < 4; r++) bm[(1 + r) * W + i] = exists[r] ? 0u : 0xffffffffu;
    }
    __syncwarp();
#pragma unroll
    for (int r = 0; r < 4; r++) {
        if (!exists[r]) continue;
        const int32_t* idx = idx_of[r / 2] + static_cast<int64_t>(row[r]) * p.T;
        const uint8_t* fl = full_of[r / 2] + static_cast<int64_t>(row[r]) * p.T;
        for (int e = lane; e < cnt[r]; e += 32) {
            const int kv = e < 32 ? kv0[r] : __ldg(&idx[e]);
            const bool full = e < 32 ? full0[r] : __ldg(&fl[e]) != 0;
            if (kv < 0 || kv >= p.T) continue;  // a corrupt index is skipped, never followed
            atomicOr(&bm[kv >> 5], 1u << (kv & 31));
            if (full) atomicOr(&bm[(1 + r) * W + (kv >> 5)], 1u << (kv & 31));
        }
    }
    __syncwarp();
    int base = 0;
    for (int w0 = 0; w0 < words; w0 += 32) {
        const int wi = w0 + lane;
        uint32_t lv = wi < words ? bm[wi] : 0u;
        const uint32_t fa = wi < words ? (bm[W + wi] & bm[2 * W + wi]) : 0u;
        const uint32_t fb = wi < words ? (bm[3 * W + wi] & bm[4 * W + wi]) : 0u;
        const int c = __popc(lv);
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        int off = base + incl - c;
        while (lv) {
            const int b = __ffs(lv) - 1;
            lv &= lv - 1;
            list[off++] = static_cast<uint16_t>((wi * 32 + b) | (((fa >> b) & 1u) << 14) | (((fb >> b) & 1u) << 15));
        }
        base += __shfl_sync(0xffffffffu, incl, 31);
    }
    __syncwarp();
    return base;
}

__device__ __forceinline__ void report(const FwdParams& p, volatile int* abort_flag, int32_t bit)
{
    *abort_flag = 1;
    atomicOr(p.status, bit);
}

// packed fp32 pairs (sm_100 f32x2 arithmetic)
__device__ __forceinline__ uint64_t f2_pack(float a, float b)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& a, float& b)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("add.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c)
{
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// 2^x for two lanes on the FMA pipe: x = j + f with j = round(x) (added in
// the float's exponent field) and f in [-1/2, 1/2], 2^f by a degree-3 minimax
// polynomial (relative error 7.5e-5, fitted by csrc/fit_exp2.py).  Returns
// exactly 0 for x < -125 (and for x = -inf), where the exponent field would
// underflow.  Valid for x <= 127.
__device__ __forceinline__ void exp2_poly_x2(uint64_t x2, float& p0, float& p1)
{
    constexpr float kRound = 12582912.0f;  // 1.5 * 2^23: x + kRound rounds x to an integer
    const uint64_t t2 = f2_add(x2, f2_pack(kRound, kRound));
    const uint64_t j2 = f2_add(t2, f2_pack(-kRound, -kRound));
    const uint64_t f2 = f2_fma(j2, f2_pack(-1.f, -1.f), x2);
    uint64_t q2 = f2_fma(f2_pack(0.0551716685295105f, 0.0551716685295105f), f2,
                         f2_pack(0.2426111251115799f, 0.2426111251115799f));
    q2 = f2_fma(q2, f2, f2_pack(0.6932609677314758f, 0.6932609677314758f));
    q2 = f2_fma(q2, f2, f2_pack(0.9999280571937561f, 0.9999280571937561f));
    float x0, x1, t0, t1, q0, q1;
    f2_unpack(x2, x0, x1);
    f2_unpack(t2, t0, t1);
    f2_unpack(q2, q0, q1);
    // the low bits of t hold j (two's complement); shifting them into the exponent field scales by 2^j
    p0 = x0 < -125.f ? 0.f : __int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23));
    p1 = x1 < -125.f ? 0.f : __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23));
}

template <int D, int BN, bool MULTI>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO, const FwdParams p,
               const __grid_constant__ HeadPatterns hp)
{
    using C = FwdCfg<D, BN>;
    constexpr int S = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem + C::kOffQ;
    uint8_t* ring = smem + C::kOffRing;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* ring_full = bars;             // [S] a K / V tile landed, or an O stage granted
    uint64_t* ring_empty = ring_full + S;   // [S] the stage may be refilled
    uint64_t* q_full = ring_empty + S;      // [2]
    uint64_t* q_empty = q_full + 2;         // [2] the slot's last S MMA of the unit is done
    uint64_t* s_full = q_empty + 2;         // [2]
    uint64_t* p_full = s_full + 2;          // [2]
    uint64_t* o_full = p_full + 2;          // [2]
    uint64_t* o_empty = o_full + 2;         // [2]
    uint64_t* o_staged = o_empty + 2;       // [2] the slot's O tile is in its ring stages (128 softmax threads)
    uint64_t* info_full = o_staged + 2;     // [2] unit-info ring: producer -> consumers
    uint64_t* info_empty = info_full + 2;   // [2] consumers (MMA, store and softmax lanes) -> producer
    uint64_t* drain = info_empty + 2;       // [1]
    uint64_t* mlx_full = drain + 1;         // [1] split unit: slot B's max and sum are in shared memory
    uint64_t* mlx_empty = mlx_full + 1;     // [1] slot A has read them
    float* mlx = reinterpret_cast<float*>(smem + C::kOffMLX);  // [2][kBM]
    uint16_t* unit_list = reinterpret_cast<uint16_t*>(smem + C::kOffList);  // [2][kMaxTiles]
    volatile int* unit_n = reinterpret_cast<volatile int*>(smem + C::kOffListN);  // [2]
    volatile int* unit_pos = unit_n + 2;  // [2] ring position of the unit's first item
    uint32_t* bitmaps = reinterpret_cast<uint32_t*>(smem + C::kOffBitmap);  // [5][kMaxTiles / 32]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;

    if (threadIdx.x == 0) {
        for (int i = 0; i < S; i++) {
            mbar_init(&ring_full[i], 1);
            mbar_init(&ring_empty[i], 1);
        }
        for (int x = 0; x < 2; x++) {
            mbar_init(&q_full[x], 1);
            mbar_init(&q_empty[x], 1);
            mbar_init(&s_full[x], 1);
            mbar_init(&p_full[x], 128);
            mbar_init(&o_full[x], 1);
            mbar_init(&o_empty[x], 128);
            mbar_init(&o_staged[x], 128);
        }
        for (int b = 0; b < 2; b++) {
            mbar_init(&info_full[b], 32);                 // every producer lane
            mbar_init(&info_empty[b], 32 + 32 + 8 * 32);  // every MMA, store and softmax lane
        }
        mbar_init(drain, 1);
        mbar_init(mlx_full, 128);
        mbar_init(mlx_empty, 128);
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
        tma_prefetch_desc(&tmO);
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const long long lim = p.timeout;
    // rows r0 .. of a plane into / out of shared memory: the token-order 3-D maps,
    // or (pattern-table kernel, grouped view) the 4-D maps at (P / n, P mod n)
    const int grp_n = MULTI ? hp.grp_n : 0;
    const int grp_s = MULTI ? hp.grp_s : 0;
    auto load_rows = [grp_n](void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int r0, int plane,
                             uint64_t pol) {
        if constexpr (MULTI) {
            if (grp_n > 0) {
                tma_load_4d(dst, map, bar, c0, r0 / grp_n, r0 % grp_n, plane, pol);
                return;
            }
        }
        tma_load_3d(dst, map, bar, c0, r0, plane, pol);
    };
    auto store_rows = [grp_n](const CUtensorMap* map, const void* src, int c0, int r0, int plane) {
        if constexpr (MULTI) {
            if (grp_n > 0) {
                tma_store_4d(map, src, c0, r0 / grp_n, r0 % grp_n, plane);
                return;
            }
        }
        tma_store_3d(map, src, c0, r0, plane);
    };
    // warp-uniform warpgroup index, so that the register split applies per branch
    const int wg = __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x) / 128, 0);

    if (wg == 0) {
        regs_dec<kRegsControl>();
    if (warp == 0) {
        // ================================================================ producer
        // Whole warp, converged: builds each unit's step list into the
        // unit-info ring, then one elected lane issues the TMA copies.
        {
            const uint64_t pol_q = policy_evict_first();
            const uint64_t pol_kv = policy_evict_last();
            auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
                return __all_sync(0xffffffffu, mbar_wait(bar, parity, lim));
            };
            int pos = 0;                // ring items issued (loads and O grants)
            int q_loads[2] = {0, 0};    // Q loads per slot (phases of q_empty)
            int q_issued[2] = {0, 0};   // of which actually issued (the test hook skips one)
            bool dead = false;
            // Take the next ring stage (bounded wait for its previous item to be released).
            auto take_stage = [&]() -> bool {
                if (!wait(&ring_empty[pos % S], ((pos / S) & 1) ^ 1)) {
                    if (lane == 0) report(p, abort_flag, ST_PRODUCER_WAIT);
                    dead = true;
                    return false;
                }
                return true;
            };
            // Build unit u's step list into ring entry k & 1 and publish it with
            // the ring position of the unit's first item.  Returns the step count.
            auto publish = [&](int u, int k, int first_pos) -> int {
                const int buf = k & 1;
                if (!wait(&info_empty[buf], ((k >> 1) & 1) ^ 1)) {
                    if (lane == 0) report(p, abort_flag, ST_PRODUCER_WAIT);
                    dead = true;
                    return 0;
                }
                const int n = build_unit_list<MULTI>(p, hp, decode_unit(p, u), BN, unit_list + buf * kMaxTiles,
                                                     bitmaps, lane);
                if (lane == 0) {
                    unit_n[buf] = n;
                    unit_pos[buf] = first_pos;
                }
                mbar_arrive(&info_full[buf]);  // every lane releases its own list writes
                return n;
            };
            int k_unit = 0;             // units of this CTA so far: ring entry k_unit & 1
            int n = unit_of(0, p.snake) < p.n_items ? publish(unit_of(0, p.snake), 0, 0) : 0;
            for (int u = unit_of(0, p.snake); u < p.n_items && !dead; u = unit_of(++k_unit, p.snake)) {
                const int buf = k_unit & 1;
                const Unit w = decode_unit(p, u);
                const uint16_t* list = unit_list + buf * kMaxTiles;
                const int u_next = unit_of(k_unit + 1, p.snake);
                // Q of the next unit into L2 now; its shared-memory load waits
                // for the slot's last S MMA of this unit
                __syncwarp();
#pragma unroll
                for (int x = 0; x < 2; x++) {
                    if (dead || slot_steps(w, n, x) == 0) continue;
                    if (!wait(&q_empty[x], (q_loads[x] & 1) ^ 1)) {
                        if (lane == 0) report(p, abort_flag, ST_PRODUCER_WAIT);
                        dead = true;
                        continue;
                    }
                    const bool skip = (p.debug_flags & 1) && x == 0 && q_loads[0] == 0;
                    if (!skip) {
                        if (elect_one()) {
                            mbar_arrive_expect_tx(&q_full[x], C::kQBytes);
                            for (int c = 0; c < D / 64; c++)
                                load_rows(sQ + x * C::kQBytes + c * C::kQPanel, &tmQ, &q_full[x], c * 64,
                                          w.qtile[x] * kBM, w.b * p.Hq + w.hq[x], pol_q);
                        }
                        __syncwarp();
                        q_issued[x]++;
                    }
                    q_loads[x]++;
                }
                const int plane = w.b * p.Hkv + w.hkv;
                if (__builtin_expect(!w.split, 1)) {
                    for (int j = 0; j < n && !dead; j++) {
                        const int kv = list[j] & 0x3fff;
#pragma unroll
                        for (int v = 0; v < 2; v++) {  // K, then V
                            if (!take_stage()) break;
                            const int st = pos % S;
                            if (elect_one()) {
                                mbar_arrive_expect_tx(&ring_full[st], C::kKVBytes);
                                for (int c = 0; c < D / 64; c++)
                                    load_rows(ring + st * C::kKVBytes + c * C::kKVPanel, v == 0 ? &tmK : &tmV,
                                              &ring_full[st], c * 64, kv * BN, plane, pol_kv);
                            }
                            __syncwarp();
                            pos++;
                        }
                        if (__any_sync(0xffffffffu, *abort_flag != 0)) dead = true;
                    }
                } else {
                    const int rounds = (n + 1) / 2;
                    for (int j = 0; j < rounds && !dead; j++) {
                        // split unit: K_A, K_B, V_A, V_B of step j while both halves have a
                        // step j, then K_A, V_A
                        const int m = j < n / 2 ? 4 : 2;
                        for (int it = 0; it < m; it++) {
                            if (!take_stage()) break;
                            const bool is_v = it >= m / 2;
                            const int kv = list[slot_entry(w, n, m == 4 ? (it & 1) : 0, j)] & 0x3fff;
                            const int st = pos % S;
                            if (elect_one()) {
                                mbar_arrive_expect_tx(&ring_full[st], C::kKVBytes);
                                for (int c = 0; c < D / 64; c++)
                                    load_rows(ring + st * C::kKVBytes + c * C::kKVPanel, is_v ? &tmV : &tmK,
                                              &ring_full[st], c * 64, kv * BN, plane, pol_kv);
                            }
                            __syncwarp();
                            pos++;
                        }
                        if (__any_sync(0xffffffffu, *abort_flag != 0)) dead = true;
                    }
                }
                // the next unit's step list, built while this unit's last steps run
                const int n_o = n > 0 ? o_slots(w) * C::kOBlocks : 0;
                const int n_next = (u_next < p.n_items && !dead) ? publish(u_next, k_unit + 1, pos + n_o) : 0;
                // the stages that will hold each slot's O tile
                for (int i = 0; i < n_o && !dead; i++) {
                    if (!take_stage()) break;
                    if (elect_one()) mbar_arrive(&ring_full[pos % S]);
                    __syncwarp();
                    pos++;
                }
                n = n_next;
                if (__any_sync(0xffffffffu, *abort_flag != 0)) dead = true;
            }
            if (__any_sync(0xffffffffu, *abort_flag != 0)) {
                // Copies still in flight land before the CTA's shared memory goes
                // away; only the newest item of each stage can be pending (an O
                // grant has already completed its phase).
                bool ok = true;
#pragma unroll
                for (int x = 0; x < 2; x++)
                    if (q_issued[x] > 0) ok &= mbar_wait(&q_full[x], (q_issued[x] - 1) & 1, lim);
                for (int i = pos > S ? pos - S : 0; i < pos; i++) ok &= mbar_wait(&ring_full[i % S], (i / S) & 1, lim);
                if (!ok && lane == 0) atomicOr(p.status, ST_DRAIN_WAIT);
            }
        }
    } else if (warp == 1) {
        // ================================================================ MMA issuer
        // The whole warp runs this loop converged (operands stay warp-uniform);
        // one elected lane issues each tcgen05.mma and tcgen05.commit.
        {
            constexpr uint32_t idesc_s = idesc_bf16_f32(kBM, BN, false, false);
            constexpr uint32_t idesc_o = idesc_bf16_f32(kBM, D, false, true);
            const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
            // Descriptors of the Q and ring bases as 32-bit halves: a slot, stage
            // or k-step moves the start address in the low half by (bytes >> 4).
            const uint64_t qd = smem_desc_sw128(smem_addr(sQ), 16, 1024);
            const uint64_t kd = smem_desc_sw128(smem_addr(ring), 16, 1024);
            const uint64_t vd = smem_desc_sw128(smem_addr(ring), C::kKVPanel, 1024);
            const uint32_t q_lo = static_cast<uint32_t>(qd), k_lo = static_cast<uint32_t>(kd);
            const uint32_t v_lo = static_cast<uint32_t>(vd), d_hi = static_cast<uint32_t>(qd >> 32);
            auto commit = [&](uint64_t* bar) {
                if (elect_one()) tc_commit(bar);
                __syncwarp();
            };
            auto issue_s = [&](int x, int stage) {
                const uint32_t a0 = q_lo + static_cast<uint32_t>((x * C::kQBytes) >> 4);
                const uint32_t b0 = k_lo + static_cast<uint32_t>((stage * C::kKVBytes) >> 4);
                if (elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < D / 16; kk++) {
                        const uint32_t qo = static_cast<uint32_t>(((kk / 4) * C::kQPanel + (kk % 4) * 32) >> 4);
                        const uint32_t ko = static_cast<uint32_t>(((kk / 4) * C::kKVPanel + (kk % 4) * 32) >> 4);
                        mma_ss(tm + x * BN, desc_from_halves(a0 + qo, d_hi), desc_from_halves(b0 + ko, d_hi), idesc_s,
                               kk > 0 ? 1u : 0u);
                    }
                }
                __syncwarp();
            };
            auto issue_pv = [&](int x, int stage, bool accumulate) {
                const uint32_t b0 = v_lo + static_cast<uint32_t>((stage * C::kKVBytes) >> 4);
                if (elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < BN / 16; kk++)
                        mma_ts(tm + 2 * BN + x * D, tm + x * BN + kk * 8,
                               desc_from_halves(b0 + static_cast<uint32_t>(kk * 128), d_hi), idesc_o,
                               (accumulate || kk > 0) ? 1u : 0u);
                }
                __syncwarp();
            };
            // every lane polls; the outcome is made warp-uniform
            auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
                return __all_sync(0xffffffffu, mbar_wait(bar, parity, lim));
            };
            int steps[2] = {0, 0};     // S/P handshakes per slot
            int units[2] = {0, 0};     // units with work per slot (phases of o_full / o_empty)
            int q_loads[2] = {0, 0};
            bool ok = true;
            int k_unit = 0;  // units of this CTA so far: ring entry k_unit & 1
            for (int u = unit_of(0, p.snake); u < p.n_items && ok; u = unit_of(++k_unit, p.snake)) {
                const int buf = k_unit & 1;
                if (!wait(&info_full[buf], (k_unit >> 1) & 1)) {
                    if (lane == 0) report(p, abort_flag, ST_MMA_WAIT);
                    ok = false;
                    break;
                }
                const int n = unit_n[buf];
                const int pos = unit_pos[buf];  // ring position of the unit's first item
                mbar_arrive(&info_empty[buf]);  // the MMA warp needs the step count and ring position
                const Unit w = decode_unit(p, u);
                if (__builtin_expect(!w.split, 1)) {
                    const int nx = w.valid[1] ? 2 : 1;
                    if (n == 0) continue;
                    // prologue: S_X(0) from K(0) at ring position pos
                    ok = wait(&ring_full[pos % S], (pos / S) & 1);
#pragma unroll
                    for (int x = 0; x < 2; x++) {
                        if (x >= nx || !ok) continue;
                        ok = wait(&q_full[x], q_loads[x] & 1);
                        if (!ok) {
                            if (lane == 0) report(p, abort_flag, ST_Q_WAIT);
                            break;
                        }
                        q_loads[x]++;
                        tc_fence_after_sync();
                        issue_s(x, pos % S);
                        commit(&s_full[x]);
                        if (n == 1) commit(&q_empty[x]);  // the slot's last read of Q
                    }
                    if (!ok) {
                        if (lane == 0) report(p, abort_flag, ST_MMA_WAIT);
                        break;
                    }
                    commit(&ring_empty[pos % S]);
                    for (int j = 0; j < n && ok; j++) {
                        const bool last = j == n - 1;
                        const int pv = pos + 2 * j + 1;  // V(j)
                        const int pk = pv + 1;           // K(j + 1)
                        ok = wait(&ring_full[pv % S], (pv / S) & 1);
#pragma unroll
                        for (int x = 0; x < 2; x++) {
                            if (x >= nx || !ok) continue;
                            ok = wait(&p_full[x], steps[x] & 1);
                            if (ok && j == 0 && units[x] > 0) ok = wait(&o_empty[x], (units[x] - 1) & 1);
                            if (!ok) break;
                            steps[x]++;
                            tc_fence_after_sync();
                            issue_pv(x, pv % S, j > 0);
                            if (last) {
                                commit(&o_full[x]);
                            } else {
                                if (x == 0 && !wait(&ring_full[pk % S], (pk / S) & 1)) {
                                    ok = false;
                                    break;
                                }
                                tc_fence_after_sync();
                                issue_s(x, pk % S);
                                commit(&s_full[x]);
                                if (j + 2 == n) commit(&q_empty[x]);  // the slot's last read of Q
                            }
                        }
                        ok = __all_sync(0xffffffffu, ok && !*abort_flag);
                        if (!ok) {
                            if (lane == 0) report(p, abort_flag, ST_MMA_WAIT);
                            break;
                        }
                        commit(&ring_empty[pv % S]);
                        if (!last) commit(&ring_empty[pk % S]);
                    }
#pragma unroll
                    for (int x = 0; x < 2; x++)
                        if (x < nx) units[x]++;
                    continue;
                }
                // split unit: each slot walks its own half of the list with its own K
                // and V; a stage is released as soon as its one reader is done
                const int ns0 = slot_steps(w, n, 0), ns1 = slot_steps(w, n, 1);
                if (ns0 == 0 && ns1 == 0) continue;
#pragma unroll
                for (int x = 0; x < 2; x++) {  // prologue: S_X of each half's first step
                    const int nsx = x ? ns1 : ns0;
                    if (nsx == 0 || !ok) continue;
                    const int k0 = pos + k_item(w, n, x, 0);
                    ok = wait(&ring_full[k0 % S], (k0 / S) & 1);
                    if (!ok) {
                        if (lane == 0) report(p, abort_flag, ST_MMA_WAIT);
                        break;
                    }
                    ok = wait(&q_full[x], q_loads[x] & 1);
                    if (!ok) {
                        if (lane == 0) report(p, abort_flag, ST_Q_WAIT);
                        break;
                    }
                    q_loads[x]++;
                    tc_fence_after_sync();
                    issue_s(x, k0 % S);
                    commit(&s_full[x]);
                    if (nsx == 1) commit(&q_empty[x]);  // the slot's last read of Q
                    commit(&ring_empty[k0 % S]);
                }
                if (!ok) break;
                for (int j = 0; j < ns0 && ok; j++) {  // slot A has at least as many steps as B
#pragma unroll
                    for (int x = 0; x < 2; x++) {
                        const int nsx = x ? ns1 : ns0;
                        if (j >= nsx || !ok) continue;
                        const int pv = pos + v_item(w, n, x, j);
                        ok = wait(&ring_full[pv % S], (pv / S) & 1);
                        ok = ok && wait(&p_full[x], steps[x] & 1);
                        if (ok && j == 0 && units[x] > 0) ok = wait(&o_empty[x], (units[x] - 1) & 1);
                        if (!ok) break;
                        steps[x]++;
                        tc_fence_after_sync();
                        issue_pv(x, pv % S, j > 0);
                        commit(&ring_empty[pv % S]);
                        if (j == nsx - 1) {
                            commit(&o_full[x]);
                        } else {
                            const int pk = pos + k_item(w, n, x, j + 1);
                            if (!wait(&ring_full[pk % S], (pk / S) & 1)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after_sync();
                            issue_s(x, pk % S);
                            commit(&s_full[x]);
                            if (j + 2 == nsx) commit(&q_empty[x]);  // the slot's last read of Q
                            commit(&ring_empty[pk % S]);
                        }
                    }
                    ok = __all_sync(0xffffffffu, ok && !*abort_flag);
                    if (!ok) {
                        if (lane == 0) report(p, abort_flag, ST_MMA_WAIT);
                        break;
                    }
                }
#pragma unroll
                for (int x = 0; x < 2; x++)
                    if ((x ? ns1 : ns0) > 0) units[x]++;
            }
            // all issued tensor-core work is finished before the memory is released
            commit(drain);
            if (!wait(drain, 0) && lane == 0) atomicOr(p.status, ST_DRAIN_WAIT);
        }
    } else if (warp == 2) {
        // ================================================================ O store
        // Lane 0 issues the TMA stores of each staged O tile and waits until they
        // have read shared memory (bulk groups are per thread), then hands the
        // stages back to the producer.  Rows past N are clipped by the map.
        bool ok = true;
        int staged[2] = {0, 0};
        int k_unit = 0;
        for (int u = unit_of(0, p.snake); u < p.n_items && ok; u = unit_of(++k_unit, p.snake)) {
            const int buf = k_unit & 1;
            ok = __all_sync(0xffffffffu, mbar_wait(&info_full[buf], (k_unit >> 1) & 1, lim));
            if (!ok) break;
            const int n = unit_n[buf];
            const int pos = unit_pos[buf];
            mbar_arrive(&info_empty[buf]);
            const Unit w = decode_unit(p, u);
            const int nx = o_slots(w);  // a split unit's O is slot A's tile
            if (n == 0) continue;
#pragma unroll
            for (int x = 0; x < 2; x++) {
                if (x >= nx || !ok) continue;
                ok = __all_sync(0xffffffffu, mbar_wait(&o_staged[x], staged[x] & 1, lim) && !*abort_flag);
                if (!ok) continue;
                staged[x]++;
                const int first = pos + 2 * n + x * C::kOBlocks;
                if (lane == 0) {
                    const int plane = w.b * p.Hq + w.hq[x];
                    for (int b = 0; b < C::kOBlocks; b++)
                        for (int c = 0; c < D / 64; c++)
                            store_rows(&tmO, ring + ((first + b) % S) * C::kKVBytes + c * C::kKVPanel, c * 64,
                                       w.qtile[x] * kBM + b * BN, plane);
                    bulk_commit_group();
                    bulk_wait_read_all();
                    for (int b = 0; b < C::kOBlocks; b++) mbar_arrive(&ring_empty[(first + b) % S]);
                }
                __syncwarp();
            }
        }
        if (lane == 0) bulk_wait_all();  // the O stores are complete
        if (!ok && lane == 0) report(p, abort_flag, ST_STORE_WAIT);
    }
    } else {
        regs_inc<kRegsSoftmax>();
        // ================================================================ softmax
        const int x = (warp - 4) / 4;    // slot
        const int quarter = warp & 3;    // tensor-memory lanes this warp may access
        const int row = quarter * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32);
        const uint32_t col_s = static_cast<uint32_t>(x * BN);
        const uint32_t col_o = static_cast<uint32_t>(2 * BN + x * D);
        int cols = max(p.sinks, p.n_global);
        int pw = p.window, ps = p.stride, pg = p.n_global;  // this slot's pattern (per unit when MULTI)
        int qlim = 0, a_lo = 0, a_hi = -1;                   // MULTI: last allowed key (causal bound), stripe
        int s_area = 0, s_cnt = 0;                           // MULTI: summary columns kv mod s_area >= s_area - s_cnt
        const uint64_t scale2 = f2_pack(p.scale_log2, p.scale_log2);
        int steps = 0, units = 0;
        int units_b = 0;   // slot A only: completed phases of o_full[1] (slot B's last PV of a unit)
        int k_split = 0;   // split units passed (phases of the max / sum hand-off)
        bool ok = true;
        int k_unit = 0;  // units of this CTA so far: ring entry k_unit & 1
        for (int u = unit_of(0, p.snake); u < p.n_items && ok; u = unit_of(++k_unit, p.snake)) {
            const int buf = k_unit & 1;
            ok = __all_sync(0xffffffffu, mbar_wait(&info_full[buf], (k_unit >> 1) & 1, lim) && !*abort_flag);
            if (!ok) break;
            const int n = unit_n[buf];
            const uint16_t* list = unit_list + buf * kMaxTiles;
            const Unit w = decode_unit(p, u);
            if (!(x == 0 ? w.valid[0] : w.valid[1])) {
                mbar_arrive(&info_empty[buf]);
                continue;
            }
            const int q = (x == 0 ? w.qtile[0] : w.qtile[1]) * kBM + row;
            // token row of query q (grouped view: t = (q mod n) s + q / n)
            const int qt = (MULTI && grp_n > 0) ? (q % grp_n) * grp_s + q / grp_n : q;
            const int64_t orow = (static_cast<int64_t>(w.b) * p.Hq + (x == 0 ? w.hq[0] : w.hq[1])) * p.N + qt;
            if constexpr (MULTI) {
                const PatternRef& pr = hp.pat[hp.head[x == 0 ? w.hq[0] : w.hq[1]]];
                if (pr.mode == 1) {
                    const int grp = q / pr.area;
                    const int need = pr.col_lo - grp;
                    a_lo = grp * pr.area + (need > 0 ? (need + pr.stride - 1) / pr.stride : 0);
                    a_hi = q - pr.shift;
                    pw = -1;
                    ps = 0;
                    pg = 0;
                    cols = 0;
                    s_cnt = 0;
                    qlim = p.N - 1;
                } else {
                    pw = pr.window;
                    ps = pr.stride;
                    pg = pr.n_global;
                    cols = max(pr.sinks, pr.n_global);
                    qlim = pr.causal ? q : p.N - 1;
                    s_area = pr.area;
                    s_cnt = pr.summary;
                    if (pr.area > 0) {
                        a_lo = (q / pr.area) * pr.area;
                        a_hi = a_lo + pr.area - 1;
                    } else {
                        a_lo = 0;
                        a_hi = -1;
                    }
                }
            }
            const bool row_all = q < pg;
            float m_ref = -INFINITY;  // running max, log2 units of the scaled score
            float l_sum = 0.f;
            const int n_self = slot_steps(w, n, x);
            const int n_b = slot_steps(w, n, 1);
            const uint16_t* slot_list = list + slot_entry(w, n, x, 0);
            for (int j = 0; j < n_self; j++) {
                const uint32_t e = slot_list[j];
                const int kv = static_cast<int>(e & 0x3fffu);
                const int kv0 = kv * BN;
                const bool masked = !((e >> (14 + x)) & 1u) || kv0 + BN > p.N;
                // Allowed columns c = kv - kv0 of this row as 32-bit words, from the
                // pattern's intervals: causal c <= dq (and kv < N), band c >= dq - window,
                // sink/global columns kv < cols, every stride-th distance, global rows.
                // Built before S arrives; applied only on partial tiles.
                uint32_t allow[BN / 32];
                if (masked) {
                    const int dq = q - kv0;
                    // MULTI: causal or not (qlim), two-sided band, stripe [a_lo, a_hi]
                    const int c_max = MULTI ? min(qlim, p.N - 1) - kv0 : min(dq, p.N - 1 - kv0);
#pragma unroll
                    for (int w = 0; w < BN / 32; w++) {
                        const int base = 32 * w;
                        uint32_t m = bits_between(0, cols - 1 - kv0 - base);
                        if (pw >= 0) m |= bits_between(dq - pw - base, MULTI ? dq + pw - base : 31);
                        if constexpr (MULTI) {
                            m |= bits_between(a_lo - kv0 - base, a_hi - kv0 - base);
                            if (s_cnt > 0) {  // the summary columns of the stripes this word touches
                                const int kb = kv0 + base;
                                for (int st = kb / s_area; st * s_area <= kb + 31; st++)
                                    m |= bits_between(st * s_area + s_area - s_cnt - kb, st * s_area + s_area - 1 - kb);
                            }
                        }
                        if (ps > 0) {
                            int r0 = dq % ps;
                            if (r0 < 0) r0 += ps;
                            int h = r0 >= base ? r0 : r0 + ((base - r0 + ps - 1) / ps) * ps;
                            for (; h < base + 32; h += ps) m |= 1u << (h - base);
                        }
                        if (row_all) m = 0xffffffffu;
                        allow[w] = m & bits_between(0, c_max - base);
                    }
                }

                ok = mbar_wait(&s_full[x], steps & 1, lim);
                ok = __all_sync(0xffffffffu, ok && !*abort_flag);
                if (!ok) break;
                tc_fence_after_sync();

                float s[BN];
                {
                    uint32_t r[BN / 32][32];
#pragma unroll
                    for (int c = 0; c < BN / 32; c++)
                        tmem_ld_32x32b_x32(tmem_addr(tmem, lane_base, col_s + 32 * c), r[c]);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < BN / 32; c++) reg_fence(r[c]);
#pragma unroll
                    for (int c = 0; c < BN; c++) s[c] = __uint_as_float(r[c / 32][c % 32]);
                }
                if (masked) {
#pragma unroll
                    for (int c = 0; c < BN; c++) s[c] = (allow[c / 32] >> (c % 32)) & 1u ? s[c] : -INFINITY;
                }

                // row max: 16 independent chains of three-input max
                float mx[16];
#pragma unroll
                for (int i = 0; i < 16; i++) mx[i] = fmax3(s[i], s[16 + i], s[32 + i]);
#pragma unroll
                for (int c = 48; c + 32 <= BN; c += 32)
#pragma unroll
                    for (int i = 0; i < 16; i++) mx[i] = fmax3(mx[i], s[c + i], s[c + 16 + i]);
                if ((BN - 48) % 32 == 16) {
#pragma unroll
                    for (int i = 0; i < 16; i++) mx[i] = fmaxf(mx[i], s[BN - 16 + i]);
                }
                const float m_tile =
                    fmax3(fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmax3(mx[6], mx[7], mx[8])),
                          fmax3(fmax3(mx[9], mx[10], mx[11]), fmax3(mx[12], mx[13], mx[14]), mx[15]), -INFINITY) *
                    p.scale_log2;
                // Rescale only when the max grows by more than 2^8: the stale
                // reference is used for O and l alike, so the result is unchanged.
                const bool grow = m_tile > m_ref + 8.f;
                float alpha = 1.f;
                if (grow) {
                    alpha = ex2_approx(m_ref - m_tile);  // 0 when m_ref = -inf
                    l_sum *= alpha;
                    m_ref = m_tile;
                }
                const float m_use = m_ref == -INFINITY ? 0.f : m_ref;
                const uint64_t neg_m = f2_pack(-m_use, -m_use);

                // p = 2^(s * scale_log2 - m): 6 of every 8 pairs on the MUFU unit,
                // 2 on the FMA pipe (exp2_poly), packed two lanes at a time.
                uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
                for (int c = 0; c < BN; c += 64) {
                    uint32_t pk[32];
#pragma unroll
                    for (int i = 0; i < 32; i++) {
                        const uint64_t x2 = f2_fma(f2_pack(s[c + 2 * i], s[c + 2 * i + 1]), scale2, neg_m);
                        float p0, p1;
                        if (((c / 2 + i) & 7) < 2) {
                            exp2_poly_x2(x2, p0, p1);
                        } else {
                            float x0, x1;
                            f2_unpack(x2, x0, x1);
                            p0 = ex2_approx(x0);
                            p1 = ex2_approx(x1);
                        }
                        acc[i & 3] = f2_add(acc[i & 3], f2_pack(p0, p1));
                        pk[i] = pack_bf16x2(p0, p1);
                    }
                    tmem_st_32x32b_x32(tmem_addr(tmem, lane_base, col_s + c / 2), pk);
                }
                {
                    float a0, a1, b0, b1, c0, c1, d0, d1;
                    f2_unpack(acc[0], a0, a1);
                    f2_unpack(acc[1], b0, b1);
                    f2_unpack(acc[2], c0, c1);
                    f2_unpack(acc[3], d0, d1);
                    l_sum += ((a0 + a1) + (b0 + b1)) + ((c0 + c1) + (d0 + d1));
                }

                if (j > 0 && __any_sync(0xffffffffu, grow)) {
                    // O_X holds every product up to tile j-1 (the commit of S_X(j) covers PV_X(j-1))
#pragma unroll
                    for (int c = 0; c < D; c += 32) {
                        uint32_t r[32];
                        tmem_ld_32x32b_x32(tmem_addr(tmem, lane_base, col_o + c), r);
                        tmem_wait_ld();
                        reg_fence(r);
#pragma unroll
                        for (int i = 0; i < 32; i++) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
                        tmem_st_32x32b_x32(tmem_addr(tmem, lane_base, col_o + c), r);
                    }
                }
                tmem_wait_st();
                tc_fence_before_sync();
                mbar_arrive(&p_full[x]);
                steps++;
            }
            // first ring item of this slot's O tile (slot A's for a split unit)
            const int o_item = unit_pos[buf] + 2 * n + (w.split ? 0 : x * C::kOBlocks);
            mbar_arrive(&info_empty[buf]);  // this lane has read the unit's steps
            if (!ok) break;

            // ---------------------------------------------------------------- epilogue
            if (__builtin_expect(!w.split, 1)) {
                if (x == 0 && n_b > 0) units_b++;
                const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
                if (n > 0) {
                    // the ring stage granted for this row's block of BN rows of O
                    const int item = o_item + row / BN;
                    ok = mbar_wait(&o_full[x], units & 1, lim);
                    ok = ok && mbar_wait(&ring_full[item % S], (item / S) & 1, lim);
                    ok = __all_sync(0xffffffffu, ok && !*abort_flag);
                    if (!ok) break;
                    uint32_t o[D / 32][32];
                    tc_fence_after_sync();
#pragma unroll
                    for (int c = 0; c < D / 32; c++) tmem_ld_32x32b_x32(tmem_addr(tmem, lane_base, col_o + 32 * c), o[c]);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < D / 32; c++) reg_fence(o[c]);
                    tc_fence_before_sync();
                    mbar_arrive(&o_empty[x]);  // O_X may now be overwritten by the next unit
                    units++;
                    // Stage the bf16 row in the granted stage, in the 128-byte-swizzled
                    // layout of a K tile (the O map's box); the store warp writes it out.
                    uint8_t* stg = ring + (item % S) * C::kKVBytes;
                    const int r = row % BN;
#pragma unroll
                    for (int c = 0; c < D; c += 8) {
                        uint4 v;
                        const uint32_t* oc = &o[c / 32][c % 32];
                        v.x = pack_bf16x2(__uint_as_float(oc[0]) * inv, __uint_as_float(oc[1]) * inv);
                        v.y = pack_bf16x2(__uint_as_float(oc[2]) * inv, __uint_as_float(oc[3]) * inv);
                        v.z = pack_bf16x2(__uint_as_float(oc[4]) * inv, __uint_as_float(oc[5]) * inv);
                        v.w = pack_bf16x2(__uint_as_float(oc[6]) * inv, __uint_as_float(oc[7]) * inv);
                        const int chunk = (c % 64) / 8;
                        *reinterpret_cast<uint4*>(stg + (c / 64) * C::kKVPanel + r * 128 + ((chunk ^ (r & 7)) * 16)) = v;
                    }
                    fence_proxy_async_smem();
                    mbar_arrive(&o_staged[x]);
                } else if (q < p.N) {
                    // no live tile for this unit: O = 0 (the slot's Q was never loaded)
                    uint4* dst = reinterpret_cast<uint4*>(p.O + orow * D);
#pragma unroll
                    for (int c = 0; c < D; c += 8) dst[c / 8] = make_uint4(0u, 0u, 0u, 0u);
                }
                if (q < p.N)
                    p.LSE[orow] = l_sum > 0.f ? (m_ref + log2f(l_sum)) * 0.69314718055994530942f : -INFINITY;
            } else if (x == 1) {
                // split unit, second half: hand this row's max and sum to slot A
                ok = mbar_wait(mlx_empty, (k_split & 1) ^ 1, lim);
                ok = __all_sync(0xffffffffu, ok && !*abort_flag);
                if (!ok) break;
                mlx[row] = m_ref;
                mlx[kBM + row] = l_sum;
                mbar_arrive(mlx_full);
                k_split++;
                if (n_self > 0) units++;  // o_full[1] completed; slot A reads O_B and frees it
            } else {
                // split unit, first half: merge both halves of the row
                ok = mbar_wait(mlx_full, k_split & 1, lim);
                ok = __all_sync(0xffffffffu, ok && !*abort_flag);
                if (!ok) break;
                const float m_b = mlx[row];
                const float l_b = mlx[kBM + row];
                mbar_arrive(mlx_empty);
                k_split++;
                const float mm = fmaxf(m_ref, m_b);
                const float wa = (n_self > 0 && m_ref != -INFINITY) ? ex2_approx(m_ref - mm) : 0.f;
                const float wb = (n_b > 0 && m_b != -INFINITY) ? ex2_approx(m_b - mm) : 0.f;
                const float lt = l_sum * wa + l_b * wb;
                const float inv = lt > 0.f ? 1.f / lt : 0.f;
                const float fa = wa * inv, fb = wb * inv;
                if (n > 0) {
                    const int item = o_item + row / BN;
                    ok = n_self == 0 || mbar_wait(&o_full[0], units & 1, lim);
                    ok = ok && (n_b == 0 || mbar_wait(&o_full[1], units_b & 1, lim));
                    ok = ok && mbar_wait(&ring_full[item % S], (item / S) & 1, lim);
                    ok = __all_sync(0xffffffffu, ok && !*abort_flag);
                    if (!ok) break;
                    tc_fence_after_sync();
                    uint8_t* stg = ring + (item % S) * C::kKVBytes;
                    const int r = row % BN;
                    const uint32_t col_a = static_cast<uint32_t>(2 * BN);
                    const uint32_t col_b = static_cast<uint32_t>(2 * BN + D);
#pragma unroll 1
                    for (int c0 = 0; c0 < D; c0 += 32) {  // one 32-column chunk of both halves at a time
                        uint32_t oa[32], ob[32];
                        // both halves are read even when one has no step (its columns then
                        // hold a stale tile, replaced by zeros below): loads under a branch
                        // cost the softmax warps registers in their main loop
                        tmem_ld_32x32b_x32(tmem_addr(tmem, lane_base, col_a + c0), oa);
                        tmem_ld_32x32b_x32(tmem_addr(tmem, lane_base, col_b + c0), ob);
                        tmem_wait_ld();
                        reg_fence(oa);
                        reg_fence(ob);
                        if (n_self == 0) {
#pragma unroll
                            for (int i = 0; i < 32; i++) oa[i] = 0u;
                        }
                        if (n_b == 0) {
#pragma unroll
                            for (int i = 0; i < 32; i++) ob[i] = 0u;
                        }
#pragma unroll
                        for (int c = 0; c < 32; c += 8) {
                            float f[8];
#pragma unroll
                            for (int i = 0; i < 8; i++)
                                f[i] = __uint_as_float(oa[c + i]) * fa + __uint_as_float(ob[c + i]) * fb;
                            uint4 v;
                            v.x = pack_bf16x2(f[0], f[1]);
                            v.y = pack_bf16x2(f[2], f[3]);
                            v.z = pack_bf16x2(f[4], f[5]);
                            v.w = pack_bf16x2(f[6], f[7]);
                            const int gc = c0 + c;  // column of O
                            const int chunk = (gc % 64) / 8;
                            *reinterpret_cast<uint4*>(stg + (gc / 64) * C::kKVPanel + r * 128 + ((chunk ^ (r & 7)) * 16)) = v;
                        }
                    }
                    tc_fence_before_sync();
                    if (n_self > 0) {
                        mbar_arrive(&o_empty[0]);
                        units++;
                    }
                    if (n_b > 0) {
                        mbar_arrive(&o_empty[1]);  // slot A's 128 threads stand in for slot B's
                        units_b++;
                    }
                    fence_proxy_async_smem();
                    mbar_arrive(&o_staged[0]);
                } else if (q < p.N) {
                    uint4* dst = reinterpret_cast<uint4*>(p.O + orow * D);
#pragma unroll
                    for (int c = 0; c < D; c += 8) dst[c / 8] = make_uint4(0u, 0u, 0u, 0u);
                }
                if (q < p.N) p.LSE[orow] = lt > 0.f ? (mm + log2f(lt)) * 0.69314718055994530942f : -INFINITY;
            }
        }
        if (!ok) report(p, abort_flag, ST_SOFTMAX_WAIT);
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

}  // namespace sa
