// fa_merge.cuh -- combine attention results over disjoint key sets.
//
// Part i holds, per query row, o_i (normalised over its own keys) and lse_i.
// Over the union of the key sets the result is
//     lse = ln sum_i exp(lse_i),    o = sum_i exp(lse_i - lse) * o_i
// -- the online softmax's rescale ("FlashAttention, Playable", EP 04),
// applied to whole partial results; it is what a sequence-parallel forward
// needs after each rank has attended to every key chunk.  HBM-bound: one warp
// per row, lane l holds elements [l*d/32, (l+1)*d/32).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "fa_decode.cuh"

namespace fa {
namespace merge {

template <typename T, int D>
__global__ void __launch_bounds__(256) fa_merge_kernel(const T* o_parts, const float* lse_parts, int parts,
                                                       int64_t rows, T* o, float* lse) {
    constexpr int kPer = D / 32;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    float big = -INFINITY;
    for (int i = 0; i < parts; ++i) big = fmaxf(big, lse_parts[i * rows + row]);
    float acc[kPer];
#pragma unroll
    for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
    if (big == -INFINITY) {  // no part has a usable key
        dec::store_slice<T, kPer>(o + row * D, lane, acc);
        if (lane == 0) lse[row] = -INFINITY;
        return;
    }
    float tot = 0.f;
    for (int i = 0; i < parts; ++i) {
        const float li = lse_parts[i * rows + row];
        if (li == -INFINITY) continue;
        const float w = exp2f((li - big) * 1.4426950408889634f);
        tot += w;
        float x[kPer];
        dec::load_slice<T, kPer>(o_parts + (i * rows + row) * D, lane, x);
#pragma unroll
        for (int e = 0; e < kPer; ++e) acc[e] = fmaf(w, x[e], acc[e]);
    }
    const float inv = 1.f / tot;
#pragma unroll
    for (int e = 0; e < kPer; ++e) acc[e] *= inv;
    dec::store_slice<T, kPer>(o + row * D, lane, acc);
    if (lane == 0) lse[row] = big + log2f(tot) * 0.69314718055994531f;
}

}  // namespace merge
}  // namespace fa
