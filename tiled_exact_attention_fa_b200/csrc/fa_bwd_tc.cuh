// fa_bwd_tc.cuh -- gradients of the attention forward on the sm_100a tensor cores.
//
// What it computes: for the forward O = softmax(scale * Q K^T [causal]) V
// with saved lse, and an upstream gradient dO,
//     P  = exp(scale * Q K^T - lse)        (recomputed, never stored)
//     dV = P^T dO,   dP = dO V^T,   dS = P * (dP - D),   D = rowsum(dO * O)
//     dQ = scale * dS K,   dK = scale * dS^T Q
// the gradient of the exact function (the pages name training as what the
// method enables -- "FlashAttention: Tiled & Fused", section "Enabling longer
// contexts in training and inference" -- and give the forward only).  Like
// the forward, no N x N matrix ever reaches HBM: each score tile lives in
// tensor memory (TMEM) and the softmax statistics come from the saved lse.
//
// Three kernels:
//   * fa_bwd_prep_kernel: per row, D = rowsum(dO * O) and L = -lse * log2(e)
//     (padded to whole 128-row blocks: L = -inf, D = 0 past the end), and the
//     row of the fp32 dQ accumulator set to zero;
//   * fa_bwd_kernel: one CTA per (head, 128-key block) walks the query blocks
//     i it can see.  With K and V resident in shared memory, per block:
//         S^T  = K Q_i^T          -> TMEM        (M = keys, N = queries)
//         dP^T = V dO_i^T         -> TMEM
//         P^T  = 2^(S^T * scale * log2 e + L_i)   (compute warps; bf16 back
//                                                  into TMEM over S^T)
//         dS^T = P^T * (dP^T - D_i)               (compute warps; bf16 into
//                                                  shared memory, once)
//         dV  += P^T dO_i         (A from TMEM)
//         dK  += dS^T Q_i         (A = the dS tile, K-major)
//         dQ_i = dS K             (A = the same tile read MN-major) -> TMEM
//     and four drain warps move each dQ_i out of TMEM into shared memory and
//     add it into the fp32 accumulator with TMA bulk reduce-adds, so every
//     product runs once: 10 units of N^2 d on the tensor core;
//   * fa_bwd_dq_convert_kernel: dQ = scale * accumulator, to bf16.
//
// Roles of fa_bwd_kernel: warps 0-7 compute (one TMEM lane = one key row per
// thread; the two warps of a lane quarter take one half of the 128 query
// columns each), warp 8 issues tcgen05.mma from one elected lane, warp 9
// streams Q_i (with its L and D slices) and dO_i with TMA, warps 10-13 drain
// dQ.  The MMA warp's order per block i keeps the tensor core fed while the
// compute warps work:
//     dV(i), S^T(i+1), dQ(i), dK(i), dP^T(i+1)
// S^T(i+1) goes over P^T(i) once dV(i) has read it (the tensor core runs one
// thread's MMAs in issue order); dQ(i) lands in the columns of dP^T(i), which
// the compute warps have read by then, and dP^T(i+1) follows once the drain
// warps have read dQ(i) -- while dK(i) runs.  Every mbarrier wait is bounded
// (status word, abort flag, drain), as in the forward.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "fa_fwd_tc.cuh"
#include "sm100_ptx.cuh"

namespace fa {
namespace bwd {

constexpr int kBlock = 128;        // rows (queries or keys) per tile
constexpr int kComputeWarps = 8;   // two per TMEM lane quarter, one half of the query columns each
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp = 9;
constexpr int kDrainWarp0 = 10;
constexpr int kDrainWarps = 4;     // one per lane quarter of the dQ tile
constexpr int kThreads = 32 * (kDrainWarp0 + kDrainWarps);
constexpr int kQSlots = 2;         // Q_i tiles in flight (each with its L and D slices)
constexpr int kStageBytes = 32 * 128;  // one drain warp's 32 rows x 32 fp32 columns
constexpr uint32_t kTmemCols = 512;
constexpr int kHeadGroup = 8;      // heads whose key blocks are interleaved in the launch order
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct Layout {
    static_assert(D == 64 || D == 128, "head dim");
    static constexpr int kHalves = D / 64;
    static constexpr int kPanelBytes = kBlock * 128;            // 128 rows x 64 bf16
    static constexpr int kTileBytes = kPanelBytes * kHalves;    // 128 x D bf16
    static constexpr int kDoSlots = D == 64 ? 2 : 1;
    static constexpr int kKOff = 0;
    static constexpr int kVOff = kTileBytes;
    static constexpr int kQOff = 2 * kTileBytes;
    static constexpr int kDoOff = kQOff + kQSlots * kTileBytes;
    static constexpr int kDsOff = kDoOff + kDoSlots * kTileBytes;    // dS^T [key][query] bf16, 2 panels
    static constexpr int kStageOff = kDsOff + 2 * kPanelBytes;       // drain staging, kStageBytes per warp
    static constexpr int kVecOff = kStageOff + kDrainWarps * kStageBytes;  // per Q slot: L[128], D[128] fp32
    static constexpr int kBarOff = kVecOff + kQSlots * 2 * kBlock * 4;
    // kv_full, q_full[Q], q_empty[Q], do_full[S], do_empty[S],
    // s_full, dp_full, p_full, ds_full, ds_free, dq_full, dq_free, done, drain
    static constexpr int kNumBars = 1 + 2 * kQSlots + 2 * kDoSlots + 9;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;         // tmem base, abort flag
    static constexpr int kBytes = kMiscOff + 16;
    static constexpr int kSmemBytes = kBytes + 1024;                // slack for 1024-byte alignment
    static constexpr uint32_t kTmemS = 0;         // S^T fp32; P^T bf16 pairs at [64h, 64h + 32)
    static constexpr uint32_t kTmemDP = 128;      // dP^T fp32, then dQ_i (M = queries)
    static constexpr uint32_t kTmemDV = 256;
    static constexpr uint32_t kTmemDK = 256 + D;
    static_assert(kSmemBytes <= 232448, "shared memory");
};

struct Params {
    __nv_bfloat16* dk;
    __nv_bfloat16* dv;
    const float* lvec;     // [bh][npad] -lse * log2(e); -inf on padding rows
    const float* dvec;     // [bh][npad] D = rowsum(dO * O); 0 on padding rows
    int* status;
    int n;                 // sequence length
    int npad;              // nblocks * 128
    int nblocks;           // ceil(n / 128)
    int bh;                // B * H
    float scale;
    float scale_log2;      // scale * log2(e)
};

// Per row of every head (padded to whole blocks): D, L, and the fp32 dQ
// accumulator row set to zero.  D / 8 threads per row, 8 elements each
// (16-byte loads of dO and O, two 16-byte zero stores).
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_prep_kernel(const __nv_bfloat16* dout, const __nv_bfloat16* o,
                                                          const float* lse, float* lvec, float* dvec,
                                                          float* dq_acc, int64_t bh, int n, int npad) {
    constexpr int kPerRow = D / 8;                   // threads per row (a power of two dividing 32)
    const int64_t prow = (static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x) / kPerRow;  // padded row
    const int part = threadIdx.x % kPerRow;
    const bool live = prow < bh * npad;              // (every lane stays for the shuffles below)
    const int64_t head = prow / npad;
    const int r = static_cast<int>(prow - head * npad);
    float acc = 0.f;
    if (live && r < n) {
        const int64_t row = head * n + r;
        const uint4 a = *reinterpret_cast<const uint4*>(dout + row * D + part * 8);
        const uint4 b = *reinterpret_cast<const uint4*>(o + row * D + part * 8);
        const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 af = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&aw[e]));
            const float2 bf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bw[e]));
            acc = fmaf(af.x, bf.x, acc);
            acc = fmaf(af.y, bf.y, acc);
        }
    }
#pragma unroll
    for (int off = kPerRow / 2; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (!live) return;
    float4* z = reinterpret_cast<float4*>(dq_acc + prow * D + part * 8);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (part == 0) {
        dvec[prow] = acc;
        lvec[prow] = r < n ? -lse[head * n + r] * kLog2e : -INFINITY;
    }
}

// dQ = scale * accumulator, rows < n of each head, to bf16 (8 values per thread).
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_dq_convert_kernel(const float* dq_acc, __nv_bfloat16* dq, int64_t bh,
                                                                int n, int npad, float scale) {
    const int64_t total = bh * n * (D / 8);
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
         t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t row = t / (D / 8);
        const int c = static_cast<int>(t - row * (D / 8)) * 8;
        const int64_t head = row / n;
        const int64_t prow = head * npad + (row - head * n);
        const float4* src = reinterpret_cast<const float4*>(dq_acc + prow * D + c);
        const float4 a = src[0], b = src[1];
        uint4 w;
        w.x = ptx::pack_bf16x2(a.x * scale, a.y * scale);
        w.y = ptx::pack_bf16x2(a.z * scale, a.w * scale);
        w.z = ptx::pack_bf16x2(b.x * scale, b.y * scale);
        w.w = ptx::pack_bf16x2(b.z * scale, b.w * scale);
        *reinterpret_cast<uint4*>(dq + row * D + c) = w;
    }
}

// D[tmem] = A[128 x D] * B[128 x D]^T over the head dim: both K-major
// 128-byte-swizzled shared-memory tiles (S^T = K Q^T, dP^T = V dO^T).
template <int D>
__device__ __forceinline__ void mma_rows_by_rows(bool leader, uint32_t d_tmem, uint32_t a_smem, uint32_t b_smem) {
    using L = Layout<D>;
    constexpr uint32_t idesc = ptx::make_idesc_bf16(kBlock, kBlock, false);
    const uint64_t ad = ptx::make_smem_desc(a_smem, 16, 1024);
    const uint64_t bd = ptx::make_smem_desc(b_smem, 16, 1024);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t off = ((ks >> 2) * L::kPanelBytes + (ks & 3) * 32) >> 4;
        if (leader) ptx::mma_ss(d_tmem, ad + off, bd + off, idesc, ks > 0);
    }
}

// Epilogue: columns [col_begin, col_begin + D/2) of a TMEM accumulator (times
// `mul`), 32 at a time, to bf16 global rows, one row per thread.
template <int D>
__device__ __forceinline__ void store_rows(uint32_t tmem_rows, __nv_bfloat16* row_ptr, bool valid, float mul,
                                           int col_begin) {
#pragma unroll
    for (int c0 = col_begin; c0 < col_begin + D / 2; c0 += 32) {
        uint32_t acc[32];
        ptx::tmem_ld32_wait(tmem_rows + c0, acc);
        uint32_t packed[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2)
            packed[e >> 1] = ptx::pack_bf16x2(__uint_as_float(acc[e]) * mul, __uint_as_float(acc[e + 1]) * mul);
        if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(row_ptr + c0);
#pragma unroll
            for (int v = 0; v < 4; ++v)
                dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
        }
    }
}

template <int D, bool kCausal>
__global__ void __launch_bounds__(kThreads, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_dq, const Params p) {
    using L = Layout<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = ptx::smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // CTA -> (key block kb, head bh): heads in groups of kHeadGroup with
    // their key blocks interleaved (their Q, dO and dQ rows stay in L2); in
    // each group key block 0 -- under the mask the one that sees the most
    // query blocks -- comes first.
    const int per_group = kHeadGroup * p.nblocks;
    const int grp = blockIdx.x / per_group;
    const int rem = blockIdx.x - grp * per_group;
    const int hg = min(kHeadGroup, p.bh - grp * kHeadGroup);
    const int kb = rem / hg;
    const int bh = grp * kHeadGroup + (rem - kb * hg);
    const int i_begin = kCausal ? kb : 0;  // query blocks that see this key block
    const int nb = p.nblocks - i_begin;

    const uint32_t bar0 = base + L::kBarOff;
    const uint32_t kv_full = bar0;
    auto q_full = [&](int s) { return bar0 + 8u * (1 + s); };
    auto q_empty = [&](int s) { return bar0 + 8u * (1 + kQSlots + s); };
    auto do_full = [&](int s) { return bar0 + 8u * (1 + 2 * kQSlots + s); };
    auto do_empty = [&](int s) { return bar0 + 8u * (1 + 2 * kQSlots + L::kDoSlots + s); };
    const uint32_t ev0 = bar0 + 8u * (1 + 2 * kQSlots + 2 * L::kDoSlots);
    const uint32_t s_full = ev0, dp_full = ev0 + 8, p_full = ev0 + 16, ds_full = ev0 + 24, ds_free = ev0 + 32,
                   dq_full = ev0 + 40, dq_free = ev0 + 48, done = ev0 + 56, drain = ev0 + 64;
    auto q_addr = [&](int s) { return base + L::kQOff + s * L::kTileBytes; };
    auto do_addr = [&](int s) { return base + L::kDoOff + s * L::kTileBytes; };
    auto vec_ptr = [&](int s) { return reinterpret_cast<const float*>(smem + L::kVecOff + s * 2 * kBlock * 4); };

    uint32_t* tmem_base_ptr = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
    const fa::tc::Sync sync{abort_flag, p.status};

    if (threadIdx.x == 0) {
        ptx::mbar_init(kv_full, 1);
        for (int s = 0; s < kQSlots; ++s) {
            ptx::mbar_init(q_full(s), 1);
            ptx::mbar_init(q_empty(s), 1);
        }
        for (int s = 0; s < L::kDoSlots; ++s) {
            ptx::mbar_init(do_full(s), 1);
            ptx::mbar_init(do_empty(s), 1);
        }
        ptx::mbar_init(s_full, 1);
        ptx::mbar_init(dp_full, 1);
        ptx::mbar_init(p_full, 32 * kComputeWarps);
        ptx::mbar_init(ds_full, 32 * kComputeWarps);
        ptx::mbar_init(ds_free, 1);
        ptx::mbar_init(dq_full, 1);
        ptx::mbar_init(dq_free, 32 * kDrainWarps);
        ptx::mbar_init(done, 1);
        ptx::mbar_init(drain, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        ptx::tmem_alloc(ptx::smem_addr(tmem_base_ptr), kTmemCols);
        ptx::tmem_relinquish();
    }
    if (warp == kLoadWarp && lane == 0) {
        ptx::prefetch_tmap(&tm_q);
        ptx::prefetch_tmap(&tm_k);
        ptx::prefetch_tmap(&tm_v);
        ptx::prefetch_tmap(&tm_do);
    }
    if (warp == kDrainWarp0 && lane == 0) ptx::prefetch_tmap(&tm_dq);
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    const uint32_t tmem = *tmem_base_ptr;

    if (warp == kLoadWarp) {
        // ------------------------------------------------------------ producer
        const bool leader = ptx::elect_one();
        const uint64_t keep = ptx::policy_evict_last();  // re-read by the head's other key blocks
        if (leader) {
            ptx::mbar_arrive_expect_tx(kv_full, 2 * L::kTileBytes);
            for (int h = 0; h < L::kHalves; ++h) {
                ptx::tma_load_3d(base + L::kKOff + h * L::kPanelBytes, &tm_k, kv_full, h * 64, kb * kBlock, bh, keep);
                ptx::tma_load_3d(base + L::kVOff + h * L::kPanelBytes, &tm_v, kv_full, h * 64, kb * kBlock, bh, keep);
            }
        }
        uint32_t nq = 0, ndo = 0;
        bool ok = true;
        for (int b = 0; b < nb && ok; ++b) {
            const int i = i_begin + b;
            const int qs = b % kQSlots;
            ok = __all_sync(0xffffffffu, fa::tc::wait_bar(sync, q_empty(qs), ((b / kQSlots) & 1) ^ 1));
            if (!ok) break;
            if (leader) {
                ptx::mbar_arrive_expect_tx(q_full(qs), L::kTileBytes + 2 * kBlock * 4);
                for (int h = 0; h < L::kHalves; ++h)
                    ptx::tma_load_3d(q_addr(qs) + h * L::kPanelBytes, &tm_q, q_full(qs), h * 64, i * kBlock, bh, keep);
                const int64_t v0 = static_cast<int64_t>(bh) * p.npad + static_cast<int64_t>(i) * kBlock;
                const uint32_t vdst = base + L::kVecOff + qs * 2 * kBlock * 4;
                ptx::bulk_load(vdst, p.lvec + v0, kBlock * 4, q_full(qs), keep);
                ptx::bulk_load(vdst + kBlock * 4, p.dvec + v0, kBlock * 4, q_full(qs), keep);
            }
            ++nq;
            const int ds = b % L::kDoSlots;
            ok = __all_sync(0xffffffffu, fa::tc::wait_bar(sync, do_empty(ds), ((b / L::kDoSlots) & 1) ^ 1));
            if (!ok) break;
            if (leader) {
                ptx::mbar_arrive_expect_tx(do_full(ds), L::kTileBytes);
                for (int h = 0; h < L::kHalves; ++h)
                    ptx::tma_load_3d(do_addr(ds) + h * L::kPanelBytes, &tm_do, do_full(ds), h * 64, i * kBlock, bh,
                                     keep);
            }
            ++ndo;
        }
        // every issued copy lands before shared memory is released
        for (uint32_t s = 0; s < static_cast<uint32_t>(kQSlots) && s < nq; ++s) {
            const uint32_t last = s + kQSlots * ((nq - 1 - s) / kQSlots);
            fa::tc::drain_bar(sync, q_full(s), (last / kQSlots) & 1);
        }
        for (uint32_t s = 0; s < static_cast<uint32_t>(L::kDoSlots) && s < ndo; ++s) {
            const uint32_t last = s + L::kDoSlots * ((ndo - 1 - s) / L::kDoSlots);
            fa::tc::drain_bar(sync, do_full(s), (last / L::kDoSlots) & 1);
        }
        fa::tc::drain_bar(sync, kv_full, 0);
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        const bool leader = ptx::elect_one();
        auto wait_all = [&](uint32_t bar, uint32_t parity) {
            return __all_sync(0xffffffffu, fa::tc::wait_bar(sync, bar, parity));
        };
        auto commit = [&](uint32_t bar) {
            if (leader) ptx::mma_commit(bar);
        };
        constexpr uint32_t idesc_dv = ptx::make_idesc_bf16(kBlock, D, true);        // A TMEM, B MN-major
        constexpr uint32_t idesc_dk = ptx::make_idesc_bf16(kBlock, D, true);        // A K-major, B MN-major
        constexpr uint32_t idesc_dq = ptx::make_idesc_bf16(kBlock, D, true, true);  // A, B MN-major
        const uint32_t ds_base = base + L::kDsOff;
        const uint64_t ds_kmajor = ptx::make_smem_desc(ds_base, 16, 1024);             // dS^T rows = keys
        const uint64_t ds_mnmajor = ptx::make_smem_desc(ds_base, L::kPanelBytes, 1024);  // dS, M = queries
        const uint64_t k_mnmajor = ptx::make_smem_desc(base + L::kKOff, L::kPanelBytes, 1024);
        auto issue_s = [&](int qs) { mma_rows_by_rows<D>(leader, tmem + L::kTmemS, base + L::kKOff, q_addr(qs)); };
        auto issue_dp = [&](int ds) {
            mma_rows_by_rows<D>(leader, tmem + L::kTmemDP, base + L::kVOff, do_addr(ds));
        };

        bool ok = wait_all(kv_full, 0) && nb > 0;
        if (ok) ok = wait_all(q_full(0), 0);
        if (ok) {
            ptx::tc_fence_after_sync();
            issue_s(0);
            commit(s_full);
            ok = wait_all(do_full(0), 0);
        }
        if (ok) {
            ptx::tc_fence_after_sync();
            issue_dp(0);
            commit(dp_full);
        }
        for (int b = 0; b < nb && ok; ++b) {
            const int qs = b % kQSlots, ds = b % L::kDoSlots;
            const uint32_t ph = b & 1;
            // dV += P^T dO_i: P^T from TMEM (16 queries = 8 columns per step;
            // queries [64h, 64h + 64) sit at columns [64h, 64h + 32)), dO_i MN-major.
            ok = wait_all(p_full, ph);
            if (!ok) break;
            ptx::tc_fence_after_sync();
            {
                const uint64_t dod = ptx::make_smem_desc(do_addr(ds), L::kPanelBytes, 1024);
#pragma unroll
                for (int ks = 0; ks < kBlock / 16; ++ks)
                    if (leader)
                        ptx::mma_ts(tmem + L::kTmemDV, tmem + L::kTmemS + 64 * (ks >> 2) + 8 * (ks & 3),
                                    dod + ((ks * 16 * 128) >> 4), idesc_dv, (b > 0 || ks > 0) ? 1u : 0u);
            }
            commit(do_empty(ds));
            // S^T(i+1) over P^T(i): issued after dV(i), executed after it
            if (b + 1 < nb) {
                ok = wait_all(q_full((b + 1) % kQSlots), ((b + 1) / kQSlots) & 1);
                if (!ok) break;
                ptx::tc_fence_after_sync();
                issue_s((b + 1) % kQSlots);
                commit(s_full);
            }
            ok = wait_all(ds_full, ph);
            if (!ok) break;
            ptx::tc_fence_after_sync();
            // dQ_i = dS K into the dP^T columns (read by the compute warps by now)
#pragma unroll
            for (int ks = 0; ks < kBlock / 16; ++ks)
                if (leader)
                    ptx::mma_ss(tmem + L::kTmemDP, ds_mnmajor + ((ks * 16 * 128) >> 4),
                                k_mnmajor + ((ks * 16 * 128) >> 4), idesc_dq, ks > 0 ? 1u : 0u);
            commit(dq_full);
            // dK += dS^T Q_i
            {
                const uint64_t qd = ptx::make_smem_desc(q_addr(qs), L::kPanelBytes, 1024);
#pragma unroll
                for (int ks = 0; ks < kBlock / 16; ++ks) {
                    const uint32_t off = ((ks >> 2) * L::kPanelBytes + (ks & 3) * 32) >> 4;
                    if (leader)
                        ptx::mma_ss(tmem + L::kTmemDK, ds_kmajor + off, qd + ((ks * 16 * 128) >> 4), idesc_dk,
                                    (b > 0 || ks > 0) ? 1u : 0u);
                }
            }
            commit(q_empty(qs));
            commit(ds_free);
            // dP^T(i+1) once dQ_i has left TMEM
            if (b + 1 < nb) {
                ok = wait_all(dq_free, ph);
                if (!ok) break;
                ok = wait_all(do_full((b + 1) % L::kDoSlots), ((b + 1) / L::kDoSlots) & 1);
                if (!ok) break;
                ptx::tc_fence_after_sync();
                issue_dp((b + 1) % L::kDoSlots);
                commit(dp_full);
            }
        }
        commit(done);
        commit(drain);
        fa::tc::drain_bar(sync, drain, 0);
        __syncwarp();
    } else if (warp < kComputeWarps) {
        // ------------------------------------------------------------ compute warps
        // Thread = key row r of the block (TMEM lane); the warp's half h of
        // the 128 query columns.
        const int q4 = warp & 3, h = warp >> 2;
        const int r = q4 * 32 + lane;
        const int key = kb * kBlock + r;
        const uint32_t lane_addr = static_cast<uint32_t>(32 * q4) << 16;
        const uint32_t t_s = tmem + lane_addr + L::kTmemS + 64 * h;
        const uint32_t t_dp = tmem + lane_addr + L::kTmemDP + 64 * h;
        // this thread's row of panel h of the dS^T tile (128-byte swizzle: 16-byte
        // chunk c of row r sits at chunk position c ^ (r % 8))
        uint8_t* ds_row = smem + L::kDsOff + h * L::kPanelBytes + r * 128;
        const float sl = p.scale_log2;
        bool ok = true;
        for (int b = 0; b < nb && ok; ++b) {
            const int i = i_begin + b;
            const uint32_t ph = b & 1;
            const float* lv = vec_ptr(b % kQSlots) + 64 * h;
            const float* dv = lv + kBlock;
            ok = __all_sync(0xffffffffu, fa::tc::wait_bar(sync, s_full, ph));
            if (!ok) break;
            ptx::tc_fence_after_sync();
            float pr[64];
            {
                uint32_t sv[64];
                ptx::tmem_ld64_wait(t_s, sv);
                const bool diag = kCausal && i == kb;  // mask keys after the query
#pragma unroll
                for (int c = 0; c < 64; c += 4) {
                    const float4 l4 = *reinterpret_cast<const float4*>(lv + c);
                    float x0, x1, x2, x3;
                    ptx::fma2(x0, x1, __uint_as_float(sv[c]), __uint_as_float(sv[c + 1]), sl, sl, l4.x, l4.y);
                    ptx::fma2(x2, x3, __uint_as_float(sv[c + 2]), __uint_as_float(sv[c + 3]), sl, sl, l4.z, l4.w);
                    pr[c] = ptx::ex2(x0);
                    pr[c + 1] = ptx::ex2(x1);
                    pr[c + 2] = ptx::ex2(x2);
                    pr[c + 3] = ptx::ex2(x3);
                    if (diag) {
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            if (r > 64 * h + c + u) pr[c + u] = 0.f;
                    }
                }
                uint32_t pk[32];
#pragma unroll
                for (int c = 0; c < 64; c += 2) pk[c >> 1] = ptx::pack_bf16x2(pr[c], pr[c + 1]);
                ptx::tmem_st32(t_s, pk);
            }
            ptx::tmem_st_wait();
            ptx::tc_fence_before_sync();
            ptx::mbar_arrive(p_full);

            ok = __all_sync(0xffffffffu, fa::tc::wait_bar(sync, dp_full, ph));
            if (ok && b > 0) ok = __all_sync(0xffffffffu, fa::tc::wait_bar(sync, ds_free, ph ^ 1));
            if (!ok) break;
            ptx::tc_fence_after_sync();
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t gv[32];
                ptx::tmem_ld32_wait(t_dp + 32 * half, gv);
                uint32_t w[16];
#pragma unroll
                for (int c = 0; c < 32; c += 4) {
                    const int cc = 32 * half + c;
                    const float4 d4 = *reinterpret_cast<const float4*>(dv + cc);
                    float e0, e1, e2, e3;
                    ptx::add2(e0, e1, __uint_as_float(gv[c]), __uint_as_float(gv[c + 1]), -d4.x, -d4.y);
                    ptx::add2(e2, e3, __uint_as_float(gv[c + 2]), __uint_as_float(gv[c + 3]), -d4.z, -d4.w);
                    ptx::mul2(e0, e1, e0, e1, pr[cc], pr[cc + 1]);
                    ptx::mul2(e2, e3, e2, e3, pr[cc + 2], pr[cc + 3]);
                    w[c >> 1] = ptx::pack_bf16x2(e0, e1);
                    w[(c >> 1) + 1] = ptx::pack_bf16x2(e2, e3);
                }
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const int chunk = 4 * half + v;  // 16-byte chunk (8 queries) of the 128-byte row
                    *reinterpret_cast<uint4*>(ds_row + ((chunk ^ (r & 7)) << 4)) =
                        make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
                }
            }
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before_sync();
            ptx::mbar_arrive(ds_full);
        }
        if (ok) ok = __all_sync(0xffffffffu, fa::tc::wait_bar(sync, done, 0));
        if (ok) {
            ptx::tc_fence_after_sync();
            const bool kvalid = key < p.n;
            const int64_t off = (static_cast<int64_t>(bh) * p.n + key) * D;
            store_rows<D>(tmem + lane_addr + L::kTmemDV, p.dv + off, kvalid, 1.f, h * (D / 2));
            store_rows<D>(tmem + lane_addr + L::kTmemDK, p.dk + off, kvalid, p.scale, h * (D / 2));
        }
    } else if (warp >= kDrainWarp0) {
        // ------------------------------------------------------------ dQ drain
        // Warp = one lane quarter (32 query rows) of dQ_i.  Columns go from
        // TMEM to registers 64 at a time; 32 at a time from registers into
        // this warp's 4 KB staging tile (128-byte swizzle) and on into the fp32
        // accumulator by a TMA reduce-add.  TMEM is released (dq_free) as soon
        // as every column is in registers or staged, so dP^T(i+1) can follow.
        const int q4 = warp & 3;
        const uint32_t t_dq = tmem + (static_cast<uint32_t>(32 * q4) << 16) + L::kTmemDP;
        const uint32_t stage = base + L::kStageOff + (warp - kDrainWarp0) * kStageBytes;
        uint8_t* stage_row = smem + L::kStageOff + (warp - kDrainWarp0) * kStageBytes + lane * 128;
        auto put = [&](const uint32_t* vals, int c0, int row0, int bhh) {
            if (lane == 0) ptx::bulk_wait_group_read0();  // the previous reduce has read the tile
            __syncwarp();
#pragma unroll
            for (int c = 0; c < 8; ++c)
                *reinterpret_cast<uint4*>(stage_row + ((c ^ (lane & 7)) << 4)) =
                    make_uint4(vals[4 * c], vals[4 * c + 1], vals[4 * c + 2], vals[4 * c + 3]);
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                ptx::tma_reduce_add_3d(&tm_dq, stage, c0, row0, bhh);
                ptx::bulk_commit_group();
            }
        };
        bool ok = true;
        for (int b = 0; b < nb && ok; ++b) {
            const int row0 = (i_begin + b) * kBlock + 32 * q4;
            ok = __all_sync(0xffffffffu, fa::tc::wait_bar(sync, dq_full, b & 1));
            if (!ok) break;
            ptx::tc_fence_after_sync();
            uint32_t lo[64];
            ptx::tmem_ld64_wait(t_dq, lo);
            if constexpr (D == 64) {
                ptx::tc_fence_before_sync();
                ptx::mbar_arrive(dq_free);
                put(lo, 0, row0, bh);
                put(lo + 32, 32, row0, bh);
            } else {
                put(lo, 0, row0, bh);
                uint32_t hi[64];
                ptx::tmem_ld64_wait(t_dq + 64, hi);
                ptx::tc_fence_before_sync();
                ptx::mbar_arrive(dq_free);
                put(lo + 32, 32, row0, bh);
                put(hi, 64, row0, bh);
                put(hi + 32, 96, row0, bh);
            }
        }
        if (lane == 0) ptx::bulk_wait_group0();  // every reduce-add has landed
        __syncwarp();
    }

    // ---------------------------------------------------------------- teardown
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    if (warp == kMmaWarp) {
        __syncwarp();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace bwd
}  // namespace fa
