// Pattern compiler: classify every (q-tile, kv-tile) of the score matrix as
// empty, partial or full, and count allowed pairs per query row.  Causal
// patterns without stripes: interval arithmetic on each tile.  Patterns
// without causality or with stripes (Area Attention, "Sparse Attention"
// glossary page, section "Anwendungen"): each row's allowed keys are a union
// of at most four intervals (two-sided band, sink/global columns, stripe, or
// the whole row for a global query), counted over each tile's columns.
//
// "Sparse Attention" glossary page, section "Ein Muster in Einsparungen
// verwandeln": a mask is split into 128 x 128 blocks so that kernels can skip
// the blocks without an allowed pair.  Here the classification is analytic:
// over a rectangle of queries [q0, q1] x keys [k0, k1] the distance q - kv
// takes every integer in [q0 - k1, q1 - k0], so each rule of the pattern
// (band, sink/global columns, global rows, stride) decides emptiness and
// fullness with a few comparisons instead of a loop over the pairs.
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <vector>

#include "../../include/sparse_attn.h"

namespace sa {

namespace {

int64_t floor_div(int64_t a, int64_t b) { return a >= 0 ? a / b : -((-a + b - 1) / b); }

// Is there a multiple of s in [a, b]?
bool has_multiple(int64_t a, int64_t b, int64_t s) { return a <= b && floor_div(b, s) * s >= a; }

struct Rect {
    int64_t q0, q1, k0, k1;  // inclusive
};

// At least one allowed pair in the rectangle.
bool any_allowed(const sa_pattern& p, const Rect& r)
{
    if (r.q1 < r.k0) return false;                          // entirely above the diagonal
    const int64_t dmin = std::max<int64_t>(0, r.q0 - r.k1);  // causal distances present: [dmin, q1 - k0]
    const int64_t dmax = r.q1 - r.k0;
    if (p.window >= 0 && dmin <= p.window) return true;      // band
    const int64_t cols = std::max(p.sinks, p.n_global);
    if (r.k0 < cols) return true;                            // sink / global column at kv = k0, q = q1
    if (p.n_global > 0 && r.q0 < p.n_global && r.k0 <= std::min<int64_t>(r.q1, p.n_global - 1))
        return true;                                         // global row
    if (p.stride > 0 && has_multiple(dmin, dmax, p.stride)) return true;
    return false;
}

// Every pair of the rectangle allowed.
bool all_allowed(const sa_pattern& p, const Rect& r)
{
    if (r.q0 < r.k1) return false;  // some pair above the diagonal
    // Pairs outside the sink/global columns and the global rows:
    const int64_t cols = std::max(p.sinks, p.n_global);
    const int64_t qa = std::max<int64_t>(r.q0, p.n_global), ka = std::max<int64_t>(r.k0, cols);
    if (qa > r.q1 || ka > r.k1) return true;
    int64_t lo = qa - r.k1;
    const int64_t hi = r.q1 - ka;
    if (p.window >= 0) lo = std::max<int64_t>(lo, int64_t(p.window) + 1);  // band covers distances <= window
    if (lo > hi) return true;
    // distances [lo, hi] remain; each must be a multiple of the stride
    if (p.stride <= 0) return false;
    if (p.stride == 1) return true;
    return lo == hi && lo % p.stride == 0;
}

// Status of a pattern: SA_OK, SA_ERR_INVALID_ARG for negative fields, or
// SA_ERR_UNSUPPORTED for a form the library does not build.
int pattern_status(const sa_pattern* p)
{
    if (!p) return SA_ERR_INVALID_ARG;
    if (p->window < -1 || p->sinks < 0 || p->stride < 0 || p->n_global < 0 || p->area < 0 || p->summary < 0)
        return SA_ERR_INVALID_ARG;
    if (p->summary > 0 && p->area == 0) return SA_ERR_INVALID_ARG;
    if (p->causal != 0 && p->causal != 1) return SA_ERR_UNSUPPORTED;
    if (p->stride > 0 && (p->causal == 0 || p->area > 0)) return SA_ERR_UNSUPPORTED;
    return SA_OK;
}

// The causal forms without stripes take the analytic per-tile classifier;
// the others the per-row interval count.
bool general_form(const sa_pattern& p) { return p.causal == 0 || p.area > 0; }

// Summary keys (kv mod A >= A - c) in [0, n].
int64_t summary_upto(int64_t n, int64_t A, int64_t c)
{
    if (n < 0) return 0;
    const int64_t m = n + 1;
    return (m / A) * c + std::max<int64_t>(0, m % A - (A - c));
}
int64_t summary_in(int64_t x, int64_t y, int64_t A, int64_t c)
{
    return x > y ? 0 : summary_upto(y, A, c) - summary_upto(x - 1, A, c);
}

// Allowed keys of row q as a union of closed intervals (no stride) and the
// periodic summary columns, clipped to [lo, hi]; returns how many keys of
// [lo, hi] it holds.
int64_t row_keys_in(const sa_pattern& p, int64_t N, int64_t q, int64_t lo, int64_t hi)
{
    if (p.causal) hi = std::min(hi, q);
    hi = std::min(hi, N - 1);
    lo = std::max<int64_t>(lo, 0);
    if (lo > hi) return 0;
    if (q < p.n_global) return hi - lo + 1;  // a global row sees every key (up to q when causal)
    int64_t a[4], b[4];
    int n = 0;
    auto add = [&](int64_t x, int64_t y) {
        x = std::max(x, lo);
        y = std::min(y, hi);
        if (x <= y) {
            a[n] = x;
            b[n] = y;
            n++;
        }
    };
    if (p.window >= 0) add(q - p.window, q + p.window);
    const int64_t cols = std::max(p.sinks, p.n_global);
    if (cols > 0) add(0, cols - 1);
    if (p.area > 0) {
        const int64_t a0 = (q / p.area) * p.area;
        add(a0, a0 + p.area - 1);
    }
    // sort (at most three intervals) and merge
    for (int i = 0; i < n; i++)
        for (int j = i + 1; j < n; j++)
            if (a[j] < a[i]) {
                std::swap(a[i], a[j]);
                std::swap(b[i], b[j]);
            }
    // summary columns not already inside the intervals: all of them in [lo, hi]
    // minus those inside each merged interval
    const int64_t A = p.area, c = std::min<int64_t>(p.summary, p.area);
    int64_t total = 0, cur_a = 0, cur_b = -1;
    if (c > 0) total += summary_in(lo, hi, A, c);
    auto close = [&]() {
        if (cur_b < cur_a) return;
        total += cur_b - cur_a + 1;
        if (c > 0) total -= summary_in(cur_a, cur_b, A, c);
    };
    for (int i = 0; i < n; i++) {
        if (a[i] > cur_b + 1 || cur_b < cur_a) {
            close();
            cur_a = a[i];
            cur_b = b[i];
        } else {
            cur_b = std::max(cur_b, b[i]);
        }
    }
    close();
    return total;
}

}  // namespace

// Allowed keys of query q (0 <= q < N): |band U columns U stride-hits|, or
// all of [0, q] for a global row.
int64_t row_pairs(const sa_pattern& p, int64_t q)
{
    if (q < p.n_global) return q + 1;
    const int64_t cols = std::min<int64_t>(std::max(p.sinks, p.n_global), q + 1);  // kv in [0, cols)
    int64_t n = cols;
    int64_t lo;  // smallest distance the band does not cover
    if (p.window >= 0) {
        const int64_t wq = std::min<int64_t>(q, p.window);  // band kv in [q - wq, q]
        const int64_t band_lo = q - wq;
        n += (wq + 1) - std::max<int64_t>(0, cols - band_lo);  // band minus its overlap with the columns
        lo = wq + 1;
    } else {
        lo = 0;
    }
    if (p.stride > 0) {
        const int64_t hi = q - cols;  // distances whose key lies right of the columns
        if (hi >= lo) n += floor_div(hi, p.stride) - floor_div(lo - 1, p.stride);
    }
    return n;
}

}  // namespace sa

extern "C" int32_t sparse_attn_num_tiles(int64_t N, int32_t block)
{
    if (N < 0 || block <= 0) return SA_ERR_INVALID_ARG;
    const int64_t T = (N + block - 1) / block;
    if (T > INT32_MAX) return SA_ERR_UNSUPPORTED;
    return static_cast<int32_t>(T);
}

extern "C" int sparse_attn_build_block_mask(const sa_pattern* pattern, int64_t N, int32_t block, sa_block_mask* out)
{
    if (!out || N < 0) return SA_ERR_INVALID_ARG;
    if (int rc = sa::pattern_status(pattern)) return rc;
    if (block != 64 && block != 128) return SA_ERR_UNSUPPORTED;
    const int64_t T64 = (N + block - 1) / block;
    if (T64 > (1 << 20)) return SA_ERR_UNSUPPORTED;
    const int32_t T = static_cast<int32_t>(T64);
    if (out->n_q_tiles < T || out->n_kv_tiles < T) return SA_ERR_BUFFER_TOO_SMALL;
    if (T > 0 && (!out->kv_count || !out->kv_index || !out->kv_full)) return SA_ERR_INVALID_ARG;

    int32_t max_row = 0;
    int64_t live = 0, nfull = 0;
    if (sa::general_form(*pattern)) {
        // per tile, the allowed keys of each of its rows within the tile's columns
        for (int32_t i = 0; i < T; i++) {
            const int64_t q0 = int64_t(i) * block, q1 = std::min<int64_t>(N, q0 + block) - 1;
            int32_t* idx = out->kv_index + int64_t(i) * T;
            uint8_t* full = out->kv_full + int64_t(i) * T;
            int32_t c = 0;
            const int32_t j_end = pattern->causal ? i : T - 1;
            for (int32_t j = 0; j <= j_end; j++) {
                const int64_t k0 = int64_t(j) * block, k1 = std::min<int64_t>(N, k0 + block) - 1;
                int64_t n = 0;
                for (int64_t q = q0; q <= q1; q++) n += sa::row_keys_in(*pattern, N, q, k0, k1);
                if (n == 0) continue;
                idx[c] = j;
                full[c] = n == (q1 - q0 + 1) * (k1 - k0 + 1) ? 1 : 0;
                nfull += full[c];
                c++;
            }
            for (int32_t t = c; t < T; t++) {
                idx[t] = -1;
                full[t] = 0;
            }
            out->kv_count[i] = c;
            live += c;
            max_row = std::max(max_row, c);
        }
        out->n_q_tiles = T;
        out->n_kv_tiles = T;
        out->block = block;
        out->max_per_row = max_row;
        out->n_live = live;
        out->n_full = nfull;
        return SA_OK;
    }
    for (int32_t i = 0; i < T; i++) {
        sa::Rect r;
        r.q0 = int64_t(i) * block;
        r.q1 = std::min<int64_t>(N, r.q0 + block) - 1;
        int32_t* idx = out->kv_index + int64_t(i) * T;
        uint8_t* full = out->kv_full + int64_t(i) * T;
        int32_t c = 0;
        for (int32_t j = 0; j <= i; j++) {  // tiles right of the diagonal hold no causal pair
            r.k0 = int64_t(j) * block;
            r.k1 = std::min<int64_t>(N, r.k0 + block) - 1;
            if (!sa::any_allowed(*pattern, r)) continue;
            idx[c] = j;
            full[c] = sa::all_allowed(*pattern, r) ? 1 : 0;
            nfull += full[c];
            c++;
        }
        for (int32_t t = c; t < T; t++) {
            idx[t] = -1;
            full[t] = 0;
        }
        out->kv_count[i] = c;
        live += c;
        max_row = std::max(max_row, c);
    }
    out->n_q_tiles = T;
    out->n_kv_tiles = T;
    out->block = block;
    out->max_per_row = max_row;
    out->n_live = live;
    out->n_full = nfull;
    return SA_OK;
}

extern "C" int sparse_attn_count_pairs(const sa_pattern* pattern, int64_t N, int64_t* pairs)
{
    if (!pattern || !pairs || N < 0) return SA_ERR_INVALID_ARG;
    if (int rc = sa::pattern_status(pattern)) return rc;
    int64_t total = 0;
    if (sa::general_form(*pattern)) {
        for (int64_t q = 0; q < N; q++) total += sa::row_keys_in(*pattern, N, q, 0, N - 1);
    } else {
        for (int64_t q = 0; q < N; q++) total += sa::row_pairs(*pattern, q);
    }
    *pairs = total;
    return SA_OK;
}

extern "C" int sparse_attn_transpose_block_mask(const sa_block_mask* rows, sa_block_mask* cols)
{
    if (!rows || !cols) return SA_ERR_INVALID_ARG;
    const int32_t T = rows->n_q_tiles;
    if (T < 0 || rows->n_kv_tiles != T) return SA_ERR_INVALID_ARG;
    if (cols->n_q_tiles < T || cols->n_kv_tiles < T) return SA_ERR_BUFFER_TOO_SMALL;
    if (T > 0 && (!rows->kv_count || !rows->kv_index || !rows->kv_full)) return SA_ERR_INVALID_ARG;
    if (T > 0 && (!cols->kv_count || !cols->kv_index || !cols->kv_full)) return SA_ERR_INVALID_ARG;
    for (int32_t c = 0; c < T; c++) cols->kv_count[c] = 0;
    int64_t live = 0, nfull = 0;
    // rows in ascending order, so every column list comes out ascending
    for (int32_t i = 0; i < T; i++) {
        const int32_t n = rows->kv_count[i];
        if (n < 0 || n > T) return SA_ERR_INVALID_ARG;
        for (int32_t e = 0; e < n; e++) {
            const int32_t c = rows->kv_index[int64_t(i) * T + e];
            if (c < 0 || c >= T) return SA_ERR_INVALID_ARG;
            const int32_t pos = cols->kv_count[c]++;
            if (pos >= T) return SA_ERR_INVALID_ARG;  // a row lists c twice
            cols->kv_index[int64_t(c) * T + pos] = i;
            cols->kv_full[int64_t(c) * T + pos] = rows->kv_full[int64_t(i) * T + e] ? 1 : 0;
            live++;
            nfull += cols->kv_full[int64_t(c) * T + pos];
        }
    }
    int32_t max_col = 0;
    for (int32_t c = 0; c < T; c++) {
        for (int32_t t = cols->kv_count[c]; t < T; t++) {
            cols->kv_index[int64_t(c) * T + t] = -1;
            cols->kv_full[int64_t(c) * T + t] = 0;
        }
        max_col = std::max(max_col, cols->kv_count[c]);
    }
    cols->n_q_tiles = T;
    cols->n_kv_tiles = T;
    cols->block = rows->block;
    cols->max_per_row = max_col;
    cols->n_live = live;
    cols->n_full = nfull;
    return SA_OK;
}

extern "C" int sparse_attn_stride_plan(const sa_pattern* pattern, int64_t N, int32_t block, sa_block_mask* pass1,
                                       sa_block_mask* pass2)
{
    if (!pattern || !pass1 || !pass2 || N < 0) return SA_ERR_INVALID_ARG;
    if (int rc = sa::pattern_status(pattern)) return rc;
    const sa_pattern pt = *pattern;
    if (pt.causal != 1 || pt.stride <= 0 || pt.area != 0) return SA_ERR_UNSUPPORTED;
    if (N % pt.stride != 0) return SA_ERR_UNSUPPORTED;
    // pass 1: the pattern without its stride, token order
    sa_pattern p1 = pt;
    p1.stride = 0;
    if (int rc = sparse_attn_build_block_mask(&p1, N, block, pass1)) return rc;
    // pass 2: grouped order P = (t mod s) * n + t / s; row P of group g allows
    // [g n + ceil((C - g) / s), P - shift]: the stride pairs outside the band
    // (q - kv > window), the sink/global columns (kv >= C) and the global rows
    const int32_t T = pass1->n_q_tiles;
    if (pass2->n_q_tiles < T || pass2->n_kv_tiles < T) return SA_ERR_BUFFER_TOO_SMALL;
    if (T > 0 && (!pass2->kv_count || !pass2->kv_index || !pass2->kv_full)) return SA_ERR_INVALID_ARG;
    const int64_t s = pt.stride, n = N / s;
    const int64_t C = std::max(pt.sinks, pt.n_global);
    const int64_t shift = pt.window >= 0 ? std::min<int64_t>(pt.window, N) / s + 1 : 0;
    std::vector<int64_t> cnt(static_cast<size_t>(T > 0 ? T : 1));
    int32_t max_row = 0;
    int64_t live = 0, nfull = 0;
    for (int32_t i = 0; i < T; i++) {
        std::fill(cnt.begin(), cnt.end(), 0);
        const int64_t q0 = int64_t(i) * block, q1 = std::min<int64_t>(N, q0 + block) - 1;
        for (int64_t P = q0; P <= q1; P++) {
            const int64_t g = P / n;
            const int64_t lo = g * n + (C > g ? (C - g + s - 1) / s : 0);
            const int64_t hi = P - shift;
            if (lo > hi) continue;
            for (int64_t c = lo / block; c <= hi / block; c++)
                cnt[c] += std::min<int64_t>(hi, c * block + block - 1) - std::max<int64_t>(lo, c * block) + 1;
        }
        int32_t* idx = pass2->kv_index + int64_t(i) * T;
        uint8_t* full = pass2->kv_full + int64_t(i) * T;
        int32_t k = 0;
        for (int32_t c = 0; c < T; c++) {
            if (cnt[c] == 0) continue;
            const int64_t k0 = int64_t(c) * block, k1 = std::min<int64_t>(N, k0 + block) - 1;
            idx[k] = c;
            full[k] = cnt[c] == (q1 - q0 + 1) * (k1 - k0 + 1) ? 1 : 0;
            nfull += full[k];
            k++;
        }
        for (int32_t e = k; e < T; e++) {
            idx[e] = -1;
            full[e] = 0;
        }
        pass2->kv_count[i] = k;
        live += k;
        max_row = std::max(max_row, k);
    }
    pass2->n_q_tiles = T;
    pass2->n_kv_tiles = T;
    pass2->block = block;
    pass2->max_per_row = max_row;
    pass2->n_live = live;
    pass2->n_full = nfull;
    return SA_OK;
}
