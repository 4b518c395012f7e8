// fa_decode_mma.cuh -- attention of new queries over a long key/value cache
// (bf16), on the warp-level tensor-core MMA.
//
// Same operation, split-KV plan, workspace and merge as fa_decode.cuh
// ("FlashAttention: Tiled & Fused", card "KV Cache: Why Generation Speeds
// Up"; online softmax of "FlashAttention, Playable", EP 04).  What changes is
// the arithmetic per key: with several queries a CUDA-core kernel spends
// about 1000 multiply-adds and a dozen shuffles per key and query group and
// runs out of issue slots below HBM speed.  Here a warp multiplies a 16-query
// tile (the group, padded with zero rows) by 8 keys at a time:
//   S (16 x 8)  = Q (16 x d) K^T      d/16 mma.m16n8k16 (bf16 in, fp32 out),
//   O (16 x d) += P (16 x 8) V (8 x d)  d/8 mma.m16n8k8,
// with P taken straight from S's accumulator registers (the C layout of the
// first product is the A layout of the second once packed to bf16), K
// fragments from ldmatrix and V fragments from ldmatrix.trans.  That is
// about six warp instructions per key instead of fifty, so the kernel is
// bound by HBM again.  Any number of queries runs in groups of 16 (a single
// query too: padded 16x, the tensor work is still far below what the loads
// take).
//
// Shared memory: a 4-stage ring of 32-key K and V tiles, each loaded by TMA
// as d/64 panels of 32 rows x 128 bytes with the 128-byte swizzle (16-byte
// chunk c of row r stored at chunk c ^ (r % 8)); the ldmatrix addresses apply
// the same XOR, so the eight rows of a matrix fall in eight different banks.
// Rows past the cache end are zero-filled by the copy (so p = 0 stays 0);
// rows of the next chunk that a tile overhangs are masked.
// Warp w of the four consumer warps takes keys 8w .. 8w + 7 of each tile.
// The running max of a row moves only when a block's max exceeds it by more
// than 8 (log2 units), so O is rarely rescaled; P <= 256 is far inside bf16.
// Every mbarrier wait is bounded; on expiry the CTA records the timeout in the
// device status word and leaves.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "fa_decode.cuh"
#include "sm100_ptx.cuh"

namespace fa {
namespace decm {

using dec::kConsumerWarps;
using dec::kProducerWarp;
using dec::kStages;
using dec::kThreads;
using dec::kTileKeys;
using dec::kWaitCycles;
using dec::kDevTimeout;

constexpr int kQ = 16;                      // queries per CTA (MMA rows)
constexpr float kMaxSlack = 8.0f;           // log2 units a block may exceed the running max by

template <int D>
struct Cfg {
    static constexpr int kPanels = D / 64;                    // 128-byte swizzle panels per row
    static constexpr int kPanelBytes = kTileKeys * 128;       // one panel of a 32-row tile
    static constexpr int kTileBytes = kPanels * kPanelBytes;  // one K (or V) tile
    static constexpr int kRingBytes = kStages * 2 * kTileBytes;
    static constexpr int kMergeBytes = kConsumerWarps * kQ * (D + 2) * 4;
    static constexpr int kBodyBytes = kRingBytes > kMergeBytes ? kRingBytes : kMergeBytes;
    static constexpr int kBarOff = (kBodyBytes + 15) & ~15;   // full[kStages], empty[kStages]
    static constexpr int kMiscOff = kBarOff + 2 * kStages * 8;  // abort flag, last-CTA flag
    static constexpr int kSmemBytes = kMiscOff + 16 + 1024;   // + slack for 1024-byte alignment
    static_assert(D == 64 || D == 128, "head dim");
};

// Byte offset, inside a tile, of the 16-byte chunk holding elements
// [d0, d0 + 8) of row r (d0 a multiple of 8).
template <int D>
__device__ __forceinline__ uint32_t tile_offset(int r, int d0) {
    const int c = (d0 & 63) >> 3;
    return static_cast<uint32_t>((d0 >> 6) * Cfg<D>::kPanelBytes + r * 128 + ((c ^ (r & 7)) << 4));
}

// ---- warp-level MMA and ldmatrix (PTX ISA: mma.sync, ldmatrix)

// C (16x8 fp32) += A (16x16 bf16, row) * B (16x8 bf16, col).
__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// C (16x8 fp32) += A (16x8 bf16, row) * B (8x8 bf16, col).
__device__ __forceinline__ void mma_1688(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5}, {%6}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(b0));
}

// Four 8x8 bf16 matrices; lane i gives the address of row i % 8 of matrix i / 8.
__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

template <int D>
__global__ void __launch_bounds__(kThreads)
    fa_decode_mma_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                         const dec::Params p) {
    using C = Cfg<D>;
    constexpr int kKSteps = D / 16;   // k-steps of Q K^T
    constexpr int kNTiles = D / 8;    // 8-column tiles of O
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = ptx::smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = static_cast<int>(blockIdx.x % static_cast<unsigned>(p.chunks));
    const int bh = static_cast<int>(blockIdx.x / static_cast<unsigned>(p.chunks));
    const int g = blockIdx.y;
    const int q0 = g * kQ;
    const int nqc = min(kQ, p.nq - q0);
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

    // per thread: rows r0 = lane / 4 and r1 = r0 + 8 of the query tile
    const int gq = lane >> 2, tq = lane & 3;
    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
    float o[kNTiles][4];
#pragma unroll
    for (int n = 0; n < kNTiles; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;

    if (warp == kProducerWarp) {
        // ------------------------------------------------------------ producer
        // One elected lane issues 2 x d/64 tensor copies per tile.
        const bool leader = ptx::elect_one();
        const uint64_t once = ptx::policy_evict_first();
        if (leader) {
            ptx::prefetch_tmap(&tm_k);
            ptx::prefetch_tmap(&tm_v);
        }
        int issued = 0;
        for (int t = 0; t < ntiles; ++t) {
            const int s = t % kStages;
            if (t >= kStages && !__all_sync(0xffffffffu, dec::wait_phase(empty(s), ((t / kStages) - 1) & 1,
                                                                        abort_flag, p.status)))
                break;
            const int row0 = key_begin + t * kTileKeys;
            if (leader) {
                ptx::mbar_arrive_expect_tx(full(s), static_cast<uint32_t>(2 * C::kTileBytes));
                const uint32_t dk = base + s * 2 * C::kTileBytes;
#pragma unroll
                for (int pn = 0; pn < C::kPanels; ++pn) {
                    ptx::tma_load_3d(dk + pn * C::kPanelBytes, &tm_k, full(s), 64 * pn, row0, bh, once);
                    ptx::tma_load_3d(dk + C::kTileBytes + pn * C::kPanelBytes, &tm_v, full(s), 64 * pn, row0, bh,
                                     once);
                }
            }
            issued = t + 1;
        }
        // every issued copy lands before the ring is reused or the CTA exits
        if (leader) {
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
        // Q fragments (A operand of m16n8k16) for every k-step; rows past the
        // group's queries are zero.
        const __nv_bfloat16* qg = static_cast<const __nv_bfloat16*>(p.q) + (static_cast<size_t>(bh) * p.nq + q0) * D;
        uint32_t qa[kKSteps][4];
        auto qword = [&](int row, int col) -> uint32_t {
            return row < nqc ? *reinterpret_cast<const uint32_t*>(qg + static_cast<size_t>(row) * D + col) : 0u;
        };
#pragma unroll
        for (int ks = 0; ks < kKSteps; ++ks) {
            qa[ks][0] = qword(gq, 16 * ks + 2 * tq);
            qa[ks][1] = qword(gq + 8, 16 * ks + 2 * tq);
            qa[ks][2] = qword(gq, 16 * ks + 8 + 2 * tq);
            qa[ks][3] = qword(gq + 8, 16 * ks + 8 + 2 * tq);
        }
        const float sl = p.scale_log2;
        // last visible key of each of this thread's rows
        const int last0 = p.causal ? p.nk - p.nq + q0 + gq : p.nk - 1;
        const int last1 = p.causal ? p.nk - p.nq + q0 + gq + 8 : p.nk - 1;
        // ldmatrix: lane i gives row i % 8 of matrix i / 8, i.e. key 8 warp + i % 8
        const int lrow = 8 * warp + (lane & 7), lmat = lane >> 3;
        for (int t = 0; t < ntiles; ++t) {
            const int s = t % kStages;
            if (!__all_sync(0xffffffffu, dec::wait_phase(full(s), (t / kStages) & 1, abort_flag, p.status))) break;
            const uint32_t kt = base + s * 2 * C::kTileBytes;
            const uint32_t vt = kt + C::kTileBytes;
            // S = Q K^T for this warp's 8 keys
            float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int ks = 0; ks < kKSteps; ks += 2) {
                uint32_t kb[4];
                ldmatrix_x4(kt + tile_offset<D>(lrow, 16 * ks + 8 * lmat), kb);  // d 16 ks .. 16 ks + 31
                mma_16816(sc, qa[ks], kb[0], kb[1]);
                mma_16816(sc, qa[ks + 1], kb[2], kb[3]);
            }
            // mask, scale to log2 units; this thread holds keys 2tq, 2tq+1 of rows r0, r1
            const int key = key_begin + t * kTileKeys + 8 * warp + 2 * tq;
            float x[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int kk = key + (i & 1);
                const int last = (i < 2) ? last0 : last1;
                x[i] = (kk < key_end && kk <= last) ? sc[i] * sl : -INFINITY;
            }
            float bm[2] = {fmaxf(x[0], x[1]), fmaxf(x[2], x[3])};
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                bm[r] = fmaxf(bm[r], __shfl_xor_sync(0xffffffffu, bm[r], 1));
                bm[r] = fmaxf(bm[r], __shfl_xor_sync(0xffffffffu, bm[r], 2));
            }
            const bool move0 = bm[0] > m[0] + kMaxSlack, move1 = bm[1] > m[1] + kMaxSlack;
            if (__any_sync(0xffffffffu, move0 || move1)) {
                const float a0 = move0 ? dec::weight(m[0], bm[0]) : 1.f;
                const float a1 = move1 ? dec::weight(m[1], bm[1]) : 1.f;
                if (move0) m[0] = bm[0];
                if (move1) m[1] = bm[1];
                l[0] *= a0;
                l[1] *= a1;
#pragma unroll
                for (int n = 0; n < kNTiles; ++n) {
                    o[n][0] *= a0;
                    o[n][1] *= a0;
                    o[n][2] *= a1;
                    o[n][3] *= a1;
                }
            }
            const float nm0 = (m[0] == -INFINITY) ? 0.f : -m[0];
            const float nm1 = (m[1] == -INFINITY) ? 0.f : -m[1];
            const float p0 = ptx::ex2(x[0] + nm0), p1 = ptx::ex2(x[1] + nm0);
            const float p2 = ptx::ex2(x[2] + nm1), p3 = ptx::ex2(x[3] + nm1);
            l[0] += p0 + p1;
            l[1] += p2 + p3;
            const uint32_t pa0 = ptx::pack_bf16x2(p0, p1), pa1 = ptx::pack_bf16x2(p2, p3);
            // O += P V: V fragments for four 8-column tiles per ldmatrix.trans
#pragma unroll
            for (int n = 0; n < kNTiles; n += 4) {
                uint32_t vb[4];
                ldmatrix_x4_trans(vt + tile_offset<D>(lrow, 8 * (n + lmat)), vb);  // d 8n .. 8n + 31
                mma_1688(o[n], pa0, pa1, vb[0]);
                mma_1688(o[n + 1], pa0, pa1, vb[1]);
                mma_1688(o[n + 2], pa0, pa1, vb[2]);
                mma_1688(o[n + 3], pa0, pa1, vb[3]);
            }
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(empty(s));
        }
        // row sums over the quad
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            l[r] += __shfl_xor_sync(0xffffffffu, l[r], 1);
            l[r] += __shfl_xor_sync(0xffffffffu, l[r], 2);
        }
    }

    // ---------------------------------------------------------------- merge
    // The ring is free once every consumer has left its loop and the producer
    // has seen its last copies land.
    __syncthreads();
    float* mw = reinterpret_cast<float*>(smem);  // [warp][kQ][D + 2]: m, l, O
    if (warp < kConsumerWarps) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            float* row = mw + (warp * kQ + gq + 8 * r) * (D + 2);
            if (tq == 0) {
                row[0] = m[r];
                row[1] = l[r];
            }
#pragma unroll
            for (int n = 0; n < kNTiles; ++n) {
                row[2 + 8 * n + 2 * tq] = o[n][2 * r];
                row[2 + 8 * n + 2 * tq + 1] = o[n][2 * r + 1];
            }
        }
    }
    __syncthreads();
    constexpr int kPer = D / 32;
    const bool single = p.chunks == 1;
    // consumer warp w combines queries w, w + 4, ... (lane = slice of O)
    for (int i = warp; i < nqc && warp < kConsumerWarps; i += kConsumerWarps) {
        float mx = -INFINITY;
        for (int w = 0; w < kConsumerWarps; ++w) mx = fmaxf(mx, mw[(w * kQ + i) * (D + 2)]);
        float lsum = 0.f, oo[kPer];
#pragma unroll
        for (int e = 0; e < kPer; ++e) oo[e] = 0.f;
        if (mx != -INFINITY) {
            for (int w = 0; w < kConsumerWarps; ++w) {
                const float* r = mw + (w * kQ + i) * (D + 2);
                const float f = dec::weight(r[0], mx);
                lsum += f * r[1];
#pragma unroll
                for (int e = 0; e < kPer; ++e) oo[e] += f * r[2 + lane * kPer + e];
            }
        }
        const int qi = q0 + i;
        if (single) {
            const float inv = 1.f / lsum;
#pragma unroll
            for (int e = 0; e < kPer; ++e) oo[e] *= inv;
            dec::store_slice<__nv_bfloat16, kPer>(
                static_cast<__nv_bfloat16*>(p.o) + (static_cast<size_t>(bh) * p.nq + qi) * D, lane, oo);
            if (lane == 0) p.lse[static_cast<size_t>(bh) * p.nq + qi] = (mx + log2f(lsum)) * 0.69314718055994531f;
        } else {
            float* dst = p.part + ((static_cast<size_t>(bh) * p.nq + qi) * p.chunks + c) * (D + 2);
            if (lane == 0) {
                dst[0] = mx;
                dst[1] = lsum;
            }
#pragma unroll
            for (int e = 0; e < kPer; ++e) dst[2 + lane * kPer + e] = oo[e];
        }
    }
    if (single) return;

    // The last CTA of this (head, query group) merges the chunks.
    __threadfence();
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
        float lsum = 0.f, oo[kPer];
#pragma unroll
        for (int e = 0; e < kPer; ++e) oo[e] = 0.f;
        for (int cc = 0; cc < p.chunks; ++cc) {
            const float* r = src + cc * (D + 2);
            const float f = dec::weight(__ldcg(r), mx);
            lsum += f * __ldcg(r + 1);
#pragma unroll
            for (int e = 0; e < kPer; ++e) oo[e] += f * __ldcg(r + 2 + lane * kPer + e);
        }
        const float inv = 1.f / lsum;
#pragma unroll
        for (int e = 0; e < kPer; ++e) oo[e] *= inv;
        dec::store_slice<__nv_bfloat16, kPer>(
            static_cast<__nv_bfloat16*>(p.o) + (static_cast<size_t>(bh) * p.nq + qi) * D, lane, oo);
        if (lane == 0) p.lse[static_cast<size_t>(bh) * p.nq + qi] = (mx + log2f(lsum)) * 0.69314718055994531f;
    }
    if (threadIdx.x == 0) p.count[bh * p.groups + g] = 0u;  // ready for the next launch
}

}  // namespace decm
}  // namespace fa
