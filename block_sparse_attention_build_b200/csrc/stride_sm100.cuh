// Stride-aware path: the data movement around its two attention passes.
//
// A pattern with a stride s admits every s-th prior token ("Sparse Attention"
// glossary page, section "Gängige Sparsity-Muster"; "Sparse-трансформеры",
// section "Основные шаблоны разреженности": a step equal to the row width of
// a flattened image).  In token order those pairs touch every tile below the
// diagonal once per row, so a block-sparse kernel executes almost all tiles
// for a few allowed pairs each.  Grouping the tokens by residue, position
//     P = (t mod s) * n + floor(t / s),   n = N / s,
// puts every pair (q, q - m s) inside one group of n consecutive positions,
// where the pairs of a query form one interval: dense tiles on the diagonal.
// The path runs the pattern without its stride in token order (pass 1), the
// stride pairs not already admitted there in the grouped order (pass 2), and
// merges the two partial softmaxes through their log-sum-exps.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

#include "sm100.cuh"

namespace sa {

// dst[plane][P][:] = src[plane][t][:] for every position P of the grouped
// order (t = (P mod n) * s + P / n); rows of D bf16, moved in 16-byte units.
template <int D>
__global__ void __launch_bounds__(256) group_by_residue_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                                int64_t planes, int N, int s, int n)
{
    constexpr int U = D * 2 / 16;  // 16-byte units per row
    const int64_t total = planes * N * U;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += int64_t(gridDim.x) * blockDim.x) {
        const int u = static_cast<int>(i % U);
        const int64_t row = i / U;
        const int P = static_cast<int>(row % N);
        const int64_t plane = row / N;
        const int g = P / n;
        const int t = (P - g * n) * s + g;
        dst[i] = src[(plane * N + t) * U + u];
    }
}

// Merge of the two passes for token row t (grouped position P of pass 2):
//   L = log(e^L1 + e^L2),  O = O1 e^(L1 - L) + O2 e^(L2 - L)
// O holds O1 on entry and the result on exit; L1 and L2 are the passes'
// natural-log LSEs (-inf for a row with no key in that pass).
template <int D>
__global__ void __launch_bounds__(256) merge_passes_kernel(__nv_bfloat16* __restrict__ O, float* __restrict__ LSE,
                                                            const __nv_bfloat16* __restrict__ O2,
                                                            const float* __restrict__ L1,
                                                            const float* __restrict__ L2, int64_t planes, int N, int s,
                                                            int n)
{
    constexpr int U = D * 2 / 16;
    const int64_t total = planes * N * U;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += int64_t(gridDim.x) * blockDim.x) {
        const int u = static_cast<int>(i % U);
        const int64_t row = i / U;
        const int t = static_cast<int>(row % N);
        const int64_t plane = row / N;
        const int64_t rp = plane * N + (t % s) * n + t / s;  // the row in pass 2's order
        const float l1 = L1[row], l2 = L2[rp];
        const float m = fmaxf(l1, l2);
        float a = 0.f, b = 0.f, L = -INFINITY;
        if (m != -INFINITY) {
            const float w1 = expf(l1 - m), w2 = expf(l2 - m);
            const float tot = w1 + w2;
            a = w1 / tot;
            b = w2 / tot;
            L = m + logf(tot);
        }
        const uint4 x = reinterpret_cast<const uint4*>(O)[i];
        const uint4 y = reinterpret_cast<const uint4*>(O2)[rp * U + u];
        const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
        uint32_t r[4];
#pragma unroll
        for (int k = 0; k < 4; k++) {
            const float2 fx = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xs[k]));
            const float2 fy = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ys[k]));
            r[k] = pack_bf16x2(a * fx.x + b * fy.x, a * fx.y + b * fy.y);
        }
        reinterpret_cast<uint4*>(O)[i] = make_uint4(r[0], r[1], r[2], r[3]);
        if (u == 0) LSE[row] = L;
    }
}

}  // namespace sa
