// fa_fwd_simt.cuh -- fp32 attention forward on the CUDA cores (FFMA).
//
// Same method as the tensor-core kernel -- K/V tiles staged in shared memory,
// scores and probabilities kept in registers, online softmax with a running
// max, running sum and rescale (FlashAttention, Playable, EP 03-04) -- in
// plain fp32 so that fp32 inputs keep fp32 accuracy (a TF32 tensor-core path
// would round the inputs to 10 mantissa bits).
//
// One CTA of 128 threads owns 16 query rows; eight threads share a row, each
// holding every eighth element of q and of the output accumulator, and a
// 32-key tile of K and V sits in shared memory.
#pragma once

#include <cstdint>

namespace fa {
namespace simt {

constexpr int kRows = 16;     // query rows per CTA
constexpr int kKeys = 32;     // keys per shared-memory tile
constexpr int kThreads = 128;
constexpr int kSplit = kThreads / kRows;  // threads per query row

struct Params {
    const float* q;
    const float* k;
    const float* v;
    float* o;
    float* lse;
    int n;
    float scale;
};

template <int D, bool kCausal>
__global__ void __launch_bounds__(kThreads)
    fa_fwd_f32_kernel(const Params p) {
    constexpr int kPer = D / kSplit;  // elements of a row each thread owns
    __shared__ __align__(16) float sk[kKeys][D];
    __shared__ __align__(16) float sv[kKeys][D];

    const int tid = threadIdx.x;
    const int r = tid / kSplit;     // row within the CTA
    const int part = tid % kSplit;  // which share of the row
    const int64_t head = blockIdx.y;
    const int row0 = blockIdx.x * kRows;
    const int row = row0 + r;
    const bool valid = row < p.n;
    const float* qh = p.q + head * p.n * D;
    const float* kh = p.k + head * p.n * D;
    const float* vh = p.v + head * p.n * D;

    float q[kPer], acc[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        q[i] = valid ? qh[static_cast<int64_t>(row) * D + part + kSplit * i] : 0.f;
        acc[i] = 0.f;
    }
    float m = -INFINITY, l = 0.f;

    const int last_key = kCausal ? min(p.n, row0 + kRows) : p.n;  // exclusive
    // K/V rows [key0, key0 + kKeys) of the next tile are read into registers
    // while the current tile is computed (zeros past the end), then staged in
    // shared memory at the top of the next iteration.
    constexpr int kLoads = kKeys * D / 4 / kThreads;
    static_assert(kKeys * D / 4 % kThreads == 0, "whole float4 loads per thread");
    float4 nk[kLoads], nv[kLoads];
    auto fetch = [&](int key0) {
#pragma unroll
        for (int j = 0; j < kLoads; ++j) {
            const int x = tid + j * kThreads;
            const int kr = x / (D / 4);
            const int kc = (x % (D / 4)) * 4;
            nk[j] = make_float4(0.f, 0.f, 0.f, 0.f);
            nv[j] = nk[j];
            if (key0 + kr < p.n) {
                const int64_t off = static_cast<int64_t>(key0 + kr) * D + kc;
                nk[j] = *reinterpret_cast<const float4*>(kh + off);
                nv[j] = *reinterpret_cast<const float4*>(vh + off);
            }
        }
    };
    if (last_key > 0) fetch(0);
    for (int key0 = 0; key0 < last_key; key0 += kKeys) {
        __syncthreads();
#pragma unroll
        for (int j = 0; j < kLoads; ++j) {
            const int x = tid + j * kThreads;
            *reinterpret_cast<float4*>(&sk[x / (D / 4)][(x % (D / 4)) * 4]) = nk[j];
            *reinterpret_cast<float4*>(&sv[x / (D / 4)][(x % (D / 4)) * 4]) = nv[j];
        }
        __syncthreads();
        if (key0 + kKeys < last_key) fetch(key0 + kKeys);

        float s[kKeys];
        float tmax = -INFINITY;
#pragma unroll
        for (int c = 0; c < kKeys; ++c) {
            float dot = 0.f;
#pragma unroll
            for (int i = 0; i < kPer; ++i) dot = fmaf(q[i], sk[c][part + kSplit * i], dot);
#pragma unroll
            for (int w = 1; w < kSplit; w <<= 1) dot += __shfl_xor_sync(0xffffffffu, dot, w);
            const int key = key0 + c;
            const bool allowed = key < p.n && (!kCausal || key <= row);
            s[c] = allowed ? dot * p.scale : -INFINITY;
            tmax = fmaxf(tmax, s[c]);
        }
        const float m_new = fmaxf(m, tmax);
        if (m_new == -INFINITY) continue;  // nothing visible yet for this row
        const float alpha = expf(m - m_new);  // 0 on the first visible tile
        float tsum = 0.f;
#pragma unroll
        for (int c = 0; c < kKeys; ++c) {
            s[c] = expf(s[c] - m_new);
            tsum += s[c];
        }
        l = l * alpha + tsum;
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            float a = acc[i] * alpha;
#pragma unroll
            for (int c = 0; c < kKeys; ++c) a = fmaf(s[c], sv[c][part + kSplit * i], a);
            acc[i] = a;
        }
        m = m_new;
    }

    if (valid) {
        const float inv_l = 1.f / l;
        float* orow = p.o + (head * p.n + row) * D;
#pragma unroll
        for (int i = 0; i < kPer; ++i) orow[part + kSplit * i] = acc[i] * inv_l;
        if (part == 0) p.lse[head * p.n + row] = m + logf(l);
    }
}

}  // namespace simt
}  // namespace fa
