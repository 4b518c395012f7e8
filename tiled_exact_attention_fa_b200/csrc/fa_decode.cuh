// fa_decode.cuh -- attention of a few new queries over a long key/value cache
// on CUDA cores (the fp32 path; bf16 runs on the warp MMA, fa_decode_mma.cuh).
//
// What it computes (per head): for nq new queries and nk cached keys (the
// new tokens' own keys are the last nq of them), O = softmax(scale * Q K^T
// [causal]) V and lse, query i sitting at position nk - nq + i and, with the
// causal mask, using keys j <= nk - nq + i ("FlashAttention: Tiled & Fused",
// card "KV Cache: Why Generation Speeds Up": past K and V are cached, each new
// token computes only its own).  Same online softmax as the forward
// (FlashAttention, Playable, EP 04): running max, running sum, rescale.
//
// B200 mapping.  With a handful of queries the work is one pass over K and V:
// about 1 FLOP per byte per query, so the bound is HBM, not the tensor core,
// and the kernel runs on CUDA cores.
//   * Split-KV: each CTA takes one (b*h, chunk of keys, group of up to 4
//     queries); chunks are sized so the grid covers the SMs several times
//     even for a single head.  A chunk's partial (m, l, O) goes to a
//     workspace; the last CTA of a head (atomic counter) merges the chunks by
//     their log-sum-exp and writes O and lse once.
//   * Warp 4 streams K and V tiles of 32 keys into a 4-stage shared-memory
//     ring with bulk async copies (one contiguous copy per tile, an mbarrier
//     per stage); warps 0-3 each take 8 keys of a tile.
//   * Lane l holds elements [l*D/32, (l+1)*D/32) of every query and of O:
//     q.k is a lane-partial dot product; the 8 partial sums of a warp's keys
//     are completed together by a transposed butterfly (9 shuffles for 8
//     keys, after which each lane quad owns one key's score, so each lane
//     computes one exponential), and P V needs no reduction at all.
// Every mbarrier wait is bounded; on expiry the CTA records the timeout in the
// device status word and leaves.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "sm100_ptx.cuh"

namespace fa {
namespace dec {

constexpr int kConsumerWarps = 4;
constexpr int kProducerWarp = 4;
constexpr int kThreads = 32 * (kConsumerWarps + 1);
constexpr int kTileKeys = 32;                              // keys per pipeline stage
constexpr int kKeysPerWarp = kTileKeys / kConsumerWarps;   // 8
constexpr int kStages = 4;
constexpr int kMaxQ = 4;                                   // queries per CTA
constexpr long long kWaitCycles = 1ll << 32;
constexpr int kDevTimeout = 1;

template <typename T, int D>
struct Cfg {
    static constexpr int kPer = D / 32;                        // row elements per lane
    static constexpr int kRowBytes = D * static_cast<int>(sizeof(T));
    static constexpr int kTileBytes = kTileKeys * kRowBytes;   // one K (or V) tile
    static constexpr int kRingBytes = kStages * 2 * kTileBytes;
    // after the last tile the ring is reused to merge the warps' partials
    static constexpr int kMergeBytes = kConsumerWarps * kMaxQ * (D + 2) * 4;
    static constexpr int kBodyBytes = kRingBytes > kMergeBytes ? kRingBytes : kMergeBytes;
    static constexpr int kBarOff = kBodyBytes;                 // full[kStages], empty[kStages]
    static constexpr int kMiscOff = kBarOff + 2 * kStages * 8; // abort flag, last-CTA flag
    static constexpr int kSmemBytes = kMiscOff + 16 + 128;     // + slack for 128-byte alignment
    static_assert(kPer >= 1 && D % 32 == 0, "head dim");
};

struct Params {
    const void* q;      // [bh][nq][D]
    const void* k;      // [bh][nk][D]
    const void* v;      // [bh][nk][D]
    void* o;            // [bh][nq][D]
    float* lse;         // [bh][nq]
    float* part;        // [bh][nq][chunks][D + 2]: m, l (log2 units), O unnormalised
    unsigned* count;    // [bh][groups]: CTAs of a (head, query group) done; zeroed before the launch
    int* status;        // device status word
    int nq, nk, chunk, chunks, groups;  // grid: (chunks * bh, groups)
    float scale_log2;   // scale * log2(e)
    int causal;
};

// Lane's kPer elements of one row, as floats.
template <typename T, int kPer>
__device__ __forceinline__ void load_slice(const T* row, int lane, float (&x)[kPer]);

template <>
__device__ __forceinline__ void load_slice<__nv_bfloat16, 4>(const __nv_bfloat16* row, int lane, float (&x)[4]) {
    const uint2 u = *reinterpret_cast<const uint2*>(row + 4 * lane);
    x[0] = __uint_as_float(u.x << 16);
    x[1] = __uint_as_float(u.x & 0xffff0000u);
    x[2] = __uint_as_float(u.y << 16);
    x[3] = __uint_as_float(u.y & 0xffff0000u);
}
template <>
__device__ __forceinline__ void load_slice<__nv_bfloat16, 2>(const __nv_bfloat16* row, int lane, float (&x)[2]) {
    const uint32_t u = *reinterpret_cast<const uint32_t*>(row + 2 * lane);
    x[0] = __uint_as_float(u << 16);
    x[1] = __uint_as_float(u & 0xffff0000u);
}
template <>
__device__ __forceinline__ void load_slice<float, 4>(const float* row, int lane, float (&x)[4]) {
    const float4 u = *reinterpret_cast<const float4*>(row + 4 * lane);
    x[0] = u.x;
    x[1] = u.y;
    x[2] = u.z;
    x[3] = u.w;
}
template <>
__device__ __forceinline__ void load_slice<float, 2>(const float* row, int lane, float (&x)[2]) {
    const float2 u = *reinterpret_cast<const float2*>(row + 2 * lane);
    x[0] = u.x;
    x[1] = u.y;
}

template <typename T, int kPer>
__device__ __forceinline__ void store_slice(T* row, int lane, const float (&x)[kPer]);

template <>
__device__ __forceinline__ void store_slice<__nv_bfloat16, 4>(__nv_bfloat16* row, int lane, const float (&x)[4]) {
    *reinterpret_cast<uint2*>(row + 4 * lane) = make_uint2(ptx::pack_bf16x2(x[0], x[1]), ptx::pack_bf16x2(x[2], x[3]));
}
template <>
__device__ __forceinline__ void store_slice<__nv_bfloat16, 2>(__nv_bfloat16* row, int lane, const float (&x)[2]) {
    *reinterpret_cast<uint32_t*>(row + 2 * lane) = ptx::pack_bf16x2(x[0], x[1]);
}
template <>
__device__ __forceinline__ void store_slice<float, 4>(float* row, int lane, const float (&x)[4]) {
    *reinterpret_cast<float4*>(row + 4 * lane) = make_float4(x[0], x[1], x[2], x[3]);
}
template <>
__device__ __forceinline__ void store_slice<float, 2>(float* row, int lane, const float (&x)[2]) {
    *reinterpret_cast<float2*>(row + 2 * lane) = make_float2(x[0], x[1]);
}

// Bounded wait; false (and the status word set) when it expires or the CTA aborts.
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* status) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!ptx::mbar_try_wait(bar, parity)) {
        if (*abort_flag) return false;
        if (clock64() - t0 > kWaitCycles) {
            *abort_flag = 1;
            atomicCAS(status, 0, kDevTimeout);
            return false;
        }
    }
    return true;
}

// f * 2^(a - b) with the conventions of empty partials (a = -inf -> 0).
__device__ __forceinline__ float weight(float a, float b) { return (a == -INFINITY) ? 0.f : ptx::ex2(a - b); }

template <typename T, int D, int NQ>
__global__ void __launch_bounds__(kThreads) fa_decode_kernel(const Params p) {
    using C = Cfg<T, D>;
    constexpr int kPer = C::kPer;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = ptx::smem_addr(smem_raw);
    const uint32_t base = (raw + 127u) & ~127u;
    uint8_t* smem = smem_raw + (base - raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = static_cast<int>(blockIdx.x % static_cast<unsigned>(p.chunks));
    const int bh = static_cast<int>(blockIdx.x / static_cast<unsigned>(p.chunks));
    const int g = blockIdx.y;
    const int q0 = g * NQ;                                   // first query of this CTA
    const int nqc = min(NQ, p.nq - q0);                      // queries of this CTA
    const int key_begin = c * p.chunk;
    const int key_end = min(p.nk, key_begin + p.chunk);
    const int ntiles = (key_end - key_begin + kTileKeys - 1) / kTileKeys;

    auto full = [&](int s) { return base + C::kBarOff + 8u * s; };
    auto empty = [&](int s) { return base + C::kBarOff + 8u * (kStages + s); };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff);
    volatile int* last_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(full(s), 1);
            ptx::mbar_init(empty(s), kConsumerWarps);
        }
        *abort_flag = 0;
        *last_flag = 0;
        ptx::fence_mbar_init();
    }
    __syncthreads();

    const size_t head_rows = static_cast<size_t>(bh) * p.nk;
    const T* kg = static_cast<const T*>(p.k) + head_rows * D;
    const T* vg = static_cast<const T*>(p.v) + head_rows * D;

    float m[NQ], l[NQ], acc[NQ][kPer];
    if (warp == kProducerWarp) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t once = ptx::policy_evict_first();  // the cache is read once
            int issued = 0;
            for (int t = 0; t < ntiles; ++t) {
                const int s = t % kStages;
                if (t >= kStages && !wait_phase(empty(s), ((t / kStages) - 1) & 1, abort_flag, p.status)) break;
                const int row0 = key_begin + t * kTileKeys;
                const int rows = min(kTileKeys, key_end - row0);
                const uint32_t bytes = static_cast<uint32_t>(rows * C::kRowBytes);
                ptx::mbar_arrive_expect_tx(full(s), 2 * bytes);
                const uint32_t dk = base + static_cast<uint32_t>(s * 2 * C::kTileBytes);
                ptx::bulk_load(dk, kg + static_cast<size_t>(row0) * D, bytes, full(s), once);
                ptx::bulk_load(dk + C::kTileBytes, vg + static_cast<size_t>(row0) * D, bytes, full(s), once);
                issued = t + 1;
            }
            // every issued copy must land before the ring is reused or the CTA exits
            for (int t = (issued > kStages ? issued - kStages : 0); t < issued; ++t) {
                const int s = t % kStages;
                const long long t0 = clock64();
                while (!ptx::mbar_try_wait(full(s), (t / kStages) & 1))
                    if (clock64() - t0 > kWaitCycles) {
                        atomicCAS(p.status, 0, kDevTimeout);
                        break;
                    }
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ consumers
        const T* qg = static_cast<const T*>(p.q) + (static_cast<size_t>(bh) * p.nq + q0) * D;
        float qr[NQ][kPer];
#pragma unroll
        for (int i = 0; i < NQ; ++i) {
            m[i] = -INFINITY;
            l[i] = 0.f;
#pragma unroll
            for (int e = 0; e < kPer; ++e) acc[i][e] = 0.f;
            if (i < nqc) {
                load_slice<T, kPer>(qg + static_cast<size_t>(i) * D, lane, qr[i]);
#pragma unroll
                for (int e = 0; e < kPer; ++e) qr[i][e] *= p.scale_log2;  // scores in log2 units
            } else {
#pragma unroll
                for (int e = 0; e < kPer; ++e) qr[i][e] = 0.f;
            }
        }
        for (int t = 0; t < ntiles; ++t) {
            const int s = t % kStages;
            if (!__all_sync(0xffffffffu, wait_phase(full(s), (t / kStages) & 1, abort_flag, p.status))) break;
            const T* kt = reinterpret_cast<const T*>(smem + s * 2 * C::kTileBytes) + warp * kKeysPerWarp * D;
            const T* vt = kt + kTileKeys * D;
            const int key0 = key_begin + t * kTileKeys + warp * kKeysPerWarp;
            // This warp's 8 keys: the lane's slice of every K and V row (V
            // rows past the cache end are zeroed so that p = 0 stays 0).  K
            // rows are taken in a lane-dependent order, slot j holding key
            // j ^ myk, so that the transposed butterfly below sends and keeps
            // the same slots on every lane and needs no selects.
            const int myk = (lane >> 2) & 7;
            float kx[kKeysPerWarp][kPer], vx[kKeysPerWarp][kPer];
#pragma unroll
            for (int j = 0; j < kKeysPerWarp; ++j) {
                load_slice<T, kPer>(kt + (j ^ myk) * D, lane, kx[j]);
                load_slice<T, kPer>(vt + j * D, lane, vx[j]);
                if (key0 + j >= key_end)
#pragma unroll
                    for (int e = 0; e < kPer; ++e) vx[j][e] = 0.f;
            }
#pragma unroll
            for (int i = 0; i < NQ; ++i) {
                if (i >= nqc) break;
                float part[kKeysPerWarp];
#pragma unroll
                for (int j = 0; j < kKeysPerWarp; ++j) {
                    float d0 = 0.f;
#pragma unroll
                    for (int e = 0; e < kPer; ++e) d0 = fmaf(qr[i][e], kx[j][e], d0);
                    part[j] = d0;
                }
                // Reduce 8 partial sums over 32 lanes with 9 shuffles.  The
                // partner across lane bit 4 has myk ^ 4, so its slot j + 4 is
                // this lane's key j ^ myk; likewise across bits 3 and 2.  After
                // three rounds lanes 4k .. 4k+3 hold the quarter sums of key
                // k, and two more complete it.
                float w4[4], w2[2], sc;
#pragma unroll
                for (int j = 0; j < 4; ++j) w4[j] = part[j] + __shfl_xor_sync(0xffffffffu, part[j + 4], 16);
#pragma unroll
                for (int j = 0; j < 2; ++j) w2[j] = w4[j] + __shfl_xor_sync(0xffffffffu, w4[j + 2], 8);
                sc = w2[0] + __shfl_xor_sync(0xffffffffu, w2[1], 4);
                sc += __shfl_xor_sync(0xffffffffu, sc, 2);
                sc += __shfl_xor_sync(0xffffffffu, sc, 1);
                // mask: past the cache, or (causal) past query i's position
                const int last = p.causal ? p.nk - p.nq + q0 + i : p.nk - 1;
                const int key = key0 + myk;
                if (key >= key_end || key > last) sc = -INFINITY;
                // online softmax over the group (8 distinct keys per lane quad)
                float gmax = fmaxf(sc, __shfl_xor_sync(0xffffffffu, sc, 4));
                gmax = fmaxf(gmax, __shfl_xor_sync(0xffffffffu, gmax, 8));
                gmax = fmaxf(gmax, __shfl_xor_sync(0xffffffffu, gmax, 16));
                const float m_new = fmaxf(m[i], gmax);
                if (m_new == -INFINITY) continue;  // no key of the group visible yet (warp-uniform)
                const float alpha = weight(m[i], m_new);
                const float pk = (sc == -INFINITY) ? 0.f : ptx::ex2(sc - m_new);
                float psum = pk + __shfl_xor_sync(0xffffffffu, pk, 4);
                psum += __shfl_xor_sync(0xffffffffu, psum, 8);
                psum += __shfl_xor_sync(0xffffffffu, psum, 16);
                l[i] = l[i] * alpha + psum;
                m[i] = m_new;
#pragma unroll
                for (int e = 0; e < kPer; ++e) acc[i][e] *= alpha;
#pragma unroll
                for (int j = 0; j < kKeysPerWarp; ++j) {
                    const float pj = __shfl_sync(0xffffffffu, pk, 4 * j);
#pragma unroll
                    for (int e = 0; e < kPer; ++e) acc[i][e] = fmaf(pj, vx[j][e], acc[i][e]);
                }
            }
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(empty(s));
        }
    }

    // ---------------------------------------------------------------- merge
    // The ring is free once every consumer has left its loop and the producer
    // has seen its last copies land.
    __syncthreads();
    float* mw = reinterpret_cast<float*>(smem);  // [warp][NQ][D + 2]: m, l, O
    if (warp < kConsumerWarps) {
#pragma unroll
        for (int i = 0; i < NQ; ++i) {
            float* r = mw + (warp * kMaxQ + i) * (D + 2);
            if (lane == 0) {
                r[0] = m[i];
                r[1] = l[i];
            }
#pragma unroll
            for (int e = 0; e < kPer; ++e) r[2 + lane * kPer + e] = acc[i][e];
        }
    }
    __syncthreads();
    const bool single = p.chunks == 1;
    // consumer warp w combines queries w, w + 4 (lane = slice of O)
    for (int i = warp; i < nqc && warp < kConsumerWarps; i += kConsumerWarps) {
        float mx = -INFINITY;
        for (int w = 0; w < kConsumerWarps; ++w) mx = fmaxf(mx, mw[(w * kMaxQ + i) * (D + 2)]);
        float lsum = 0.f, o[kPer];
#pragma unroll
        for (int e = 0; e < kPer; ++e) o[e] = 0.f;
        if (mx != -INFINITY) {
            for (int w = 0; w < kConsumerWarps; ++w) {
                const float* r = mw + (w * kMaxQ + i) * (D + 2);
                const float f = weight(r[0], mx);
                lsum += f * r[1];
#pragma unroll
                for (int e = 0; e < kPer; ++e) o[e] += f * r[2 + lane * kPer + e];
            }
        }
        const int qi = q0 + i;
        if (single) {
            const float inv = 1.f / lsum;
#pragma unroll
            for (int e = 0; e < kPer; ++e) o[e] *= inv;
            store_slice<T, kPer>(static_cast<T*>(p.o) + (static_cast<size_t>(bh) * p.nq + qi) * D, lane, o);
            if (lane == 0) p.lse[static_cast<size_t>(bh) * p.nq + qi] = (mx + log2f(lsum)) * 0.69314718055994531f;
        } else {
            float* dst = p.part + ((static_cast<size_t>(bh) * p.nq + qi) * p.chunks + c) * (D + 2);
            if (lane == 0) {
                dst[0] = mx;
                dst[1] = lsum;
            }
#pragma unroll
            for (int e = 0; e < kPer; ++e) dst[2 + lane * kPer + e] = o[e];
        }
    }
    if (single) return;

    // The last CTA of this (head, query group) merges the chunks.
    __threadfence();  // this CTA's partials are visible before it is counted
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned done = atomicAdd(p.count + bh * p.groups + g, 1u);
        *last_flag = (done == static_cast<unsigned>(p.chunks - 1)) ? 1 : 0;
    }
    __syncthreads();
    if (!*last_flag) return;
    __threadfence();
    for (int i = warp; i < nqc && warp < kConsumerWarps; i += kConsumerWarps) {
        const int qi = q0 + i;
        const float* src = p.part + (static_cast<size_t>(bh) * p.nq + qi) * p.chunks * (D + 2);
        float mx = -INFINITY;
        for (int cc = 0; cc < p.chunks; ++cc) mx = fmaxf(mx, __ldcg(src + cc * (D + 2)));
        float lsum = 0.f, o[kPer];
#pragma unroll
        for (int e = 0; e < kPer; ++e) o[e] = 0.f;
        for (int cc = 0; cc < p.chunks; ++cc) {
            const float* r = src + cc * (D + 2);
            const float f = weight(__ldcg(r), mx);
            lsum += f * __ldcg(r + 1);
#pragma unroll
            for (int e = 0; e < kPer; ++e) o[e] += f * __ldcg(r + 2 + lane * kPer + e);
        }
        const float inv = 1.f / lsum;
#pragma unroll
        for (int e = 0; e < kPer; ++e) o[e] *= inv;
        store_slice<T, kPer>(static_cast<T*>(p.o) + (static_cast<size_t>(bh) * p.nq + qi) * D, lane, o);
        if (lane == 0) p.lse[static_cast<size_t>(bh) * p.nq + qi] = (mx + log2f(lsum)) * 0.69314718055994531f;
    }
    if (threadIdx.x == 0) p.count[bh * p.groups + g] = 0u;  // ready for the next launch
}

}  // namespace dec
}  // namespace fa
