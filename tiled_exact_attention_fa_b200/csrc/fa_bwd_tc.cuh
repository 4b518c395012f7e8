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
//   * fa_bwd_dot_kernel: D = rowsum(dO * O), one warp per row;
//   * fa_bwd_dq_kernel: one CTA per (head, 128-row query block) walks the KV
//     blocks: S = Q K_j^T and dP = dO V_j^T into TMEM, the compute warps turn
//     them into dS (bf16, into free TMEM columns), then dQ += dS K_j in TMEM;
//   * fa_bwd_dkdv_kernel: one CTA per (head, 128-key block) walks the query
//     blocks: S^T = K Q_i^T and dP^T = V dO_i^T into TMEM, the compute warps
//     write P^T and dS^T (bf16) over them, then dV += P^T dO_i and
//     dK += dS^T Q_i in TMEM.
// S and dP are computed in both kernels (so dQ needs no atomics across
// CTAs); that is 14 instead of 10 units of N^2 d work.  Roles per CTA: warps
// 0-7 compute (one TMEM lane = one row per thread; the two warps of a lane
// quarter take one half of the 128 columns each), warp 8 issues
// tcgen05.mma from one elected lane, warp 9 streams tiles with TMA through a
// 4-slot shared-memory ring.  All operand forms are the forward's: K-major
// shared-memory operands (Q, K, V, dO with d contiguous), MN-major B operands
// for the products over rows (K, Q, dO as [rows][d]), and A from TMEM.
// Every mbarrier wait is bounded (status word, abort flag, drain), as in the
// forward.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "fa_fwd_tc.cuh"
#include "sm100_ptx.cuh"

namespace fa {
namespace bwd {

constexpr int kBlock = 128;       // rows (queries or keys) per tile
constexpr int kComputeWarps = 8;  // two per TMEM lane quarter, one half of the columns each
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp = 9;
constexpr int kThreads = 320;
constexpr int kSlots = 4;         // streamed tiles in flight
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct Layout {
    static_assert(D == 64 || D == 128, "head dim");
    static constexpr int kHalves = D / 64;
    static constexpr int kPanelBytes = kBlock * 128;
    static constexpr int kTileBytes = kPanelBytes * kHalves;
    static constexpr int kAOff = 0;                                 // resident tile A (Q or K)
    static constexpr int kBOff = kTileBytes;                        // resident tile B (dO or V)
    static constexpr int kRingOff = 2 * kTileBytes;
    static constexpr int kBarOff = kRingOff + kSlots * kTileBytes;
    // a_full, b_full, full[S], empty[S], s_full, p_full, done, drain, sdp_free, p_full_odd
    static constexpr int kNumBars = 2 + 2 * kSlots + 6;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;         // tmem base, abort flag
    static constexpr int kVecOff = (kMiscOff + 16 + 15) & ~15;      // float[2][kBlock] (dK/dV kernel)
    static constexpr int kBytes = kVecOff + 2 * kBlock * 4;
    static constexpr int kSmemBytes = kBytes + 1024;
    static constexpr uint32_t kTmemS = 0;        // S or S^T; P^T / dS over its first 64 columns
    static constexpr uint32_t kTmemDP = 128;     // dP or dP^T; dS^T over its first 64 columns
    static constexpr uint32_t kTmemAcc0 = 256;   // dQ, or dV
    static constexpr uint32_t kTmemAcc1 = 256 + D;  // dK
    static constexpr uint32_t kTmemDS = 384;         // dS of the dQ kernel: two buffers of 64 columns
};

struct Params {
    __nv_bfloat16* out0;   // dQ (dq kernel) or dV (dkdv kernel)
    __nv_bfloat16* out1;   // dK (dkdv kernel)
    const float* lse;      // [bh][n] natural log, from the forward
    const float* dsum;     // [bh][n] D = rowsum(dO * O)
    int* status;
    int n;
    int nblocks;           // ceil(n / 128)
    float scale;
    float scale_log2;      // scale * log2(e)
};

// D = rowsum(dO * O) in fp32: one warp per row, lane l takes a d/32 slice.
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_dot_kernel(const __nv_bfloat16* dout, const __nv_bfloat16* o,
                                                         float* dsum, int64_t rows) {
    const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    constexpr int kPer = D / 32;
    const __nv_bfloat16* a = dout + row * D + lane * kPer;
    const __nv_bfloat16* b = o + row * D + lane * kPer;
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < kPer; ++e) acc = fmaf(__bfloat162float(a[e]), __bfloat162float(b[e]), acc);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) dsum[row] = acc;
}

// Shared pieces of the two main kernels.
template <int D>
struct Common {
    using L = Layout<D>;
    uint32_t base;
    uint32_t bar0;
    __device__ uint32_t a_full() const { return bar0; }
    __device__ uint32_t b_full() const { return bar0 + 8u; }
    __device__ uint32_t full(int s) const { return bar0 + 8u * (2 + s); }
    __device__ uint32_t empty(int s) const { return bar0 + 8u * (2 + kSlots + s); }
    __device__ uint32_t s_full() const { return bar0 + 8u * (2 + 2 * kSlots); }
    __device__ uint32_t p_full() const { return bar0 + 8u * (3 + 2 * kSlots); }
    __device__ uint32_t done() const { return bar0 + 8u * (4 + 2 * kSlots); }
    __device__ uint32_t drain() const { return bar0 + 8u * (5 + 2 * kSlots); }
    __device__ uint32_t sdp_free() const { return bar0 + 8u * (6 + 2 * kSlots); }
    // the dQ kernel's dS(j) is signalled on p_full for even j and on this one
    // for odd j: the compute warps may finish dS(j+1) before the MMA warp has
    // observed dS(j), and one barrier would then complete two phases unseen
    __device__ uint32_t p_full_odd() const { return bar0 + 8u * (7 + 2 * kSlots); }
    __device__ uint32_t p_full_of(int j) const { return (j & 1) ? p_full_odd() : p_full(); }
    __device__ uint32_t slot_addr(int s) const { return base + L::kRingOff + s * L::kTileBytes; }
};

// Producer: the two resident tiles of the unit (rows `row0` of maps ra, rb),
// then, for each streamed block b in [b_begin, b_end), tile b of map sa and
// tile b of map sb through the ring.  Waits until every copy has landed.
template <int D>
__device__ void produce(const Common<D>& c, const fa::tc::Sync& sync, const CUtensorMap* ra,
                        const CUtensorMap* rb, int row0, const CUtensorMap* sa, const CUtensorMap* sb, int b_begin,
                        int b_end, int bh) {
    using L = Layout<D>;
    const bool leader = ptx::elect_one();
    const uint64_t keep = ptx::policy_evict_last();
    if (leader) {
        ptx::mbar_arrive_expect_tx(c.a_full(), L::kTileBytes);
        for (int h = 0; h < L::kHalves; ++h)
            ptx::tma_load_3d(c.base + L::kAOff + h * L::kPanelBytes, ra, c.a_full(), h * 64, row0, bh, keep);
        ptx::mbar_arrive_expect_tx(c.b_full(), L::kTileBytes);
        for (int h = 0; h < L::kHalves; ++h)
            ptx::tma_load_3d(c.base + L::kBOff + h * L::kPanelBytes, rb, c.b_full(), h * 64, row0, bh, keep);
    }
    int slot = 0;
    uint32_t phase = 0, nloads = 0;
    bool ok = true;
    for (int b = b_begin; b < b_end && ok; ++b) {
        for (int which = 0; which < 2 && ok; ++which) {
            ok = __all_sync(0xffffffffu, fa::tc::wait_bar(sync, c.empty(slot), phase ^ 1));
            if (!ok) break;
            if (leader) {
                ptx::mbar_arrive_expect_tx(c.full(slot), L::kTileBytes);
                const CUtensorMap* m = which == 0 ? sa : sb;
                for (int h = 0; h < L::kHalves; ++h)
                    ptx::tma_load_3d(c.slot_addr(slot) + h * L::kPanelBytes, m, c.full(slot), h * 64, b * kBlock, bh,
                                     keep);
            }
            ++nloads;
            if (++slot == kSlots) {
                slot = 0;
                phase ^= 1;
            }
        }
    }
    // every issued copy lands before shared memory is released
    for (uint32_t s = 0; s < static_cast<uint32_t>(kSlots) && s < nloads; ++s) {
        const uint32_t last = s + kSlots * ((nloads - 1 - s) / kSlots);
        fa::tc::drain_bar(sync, c.full(s), (last / kSlots) & 1);
    }
    fa::tc::drain_bar(sync, c.a_full(), 0);
    fa::tc::drain_bar(sync, c.b_full(), 0);
    __syncwarp();
}

// 8 MMAs of K = 16 over the head dim: D[tmem] = A[128 x D] * B[128 x D]^T,
// both K-major 128-byte-swizzled shared-memory tiles.
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

// 8 MMAs of K = 16 over 128 rows: D[tmem, 128 x D] (+)= A[tmem, 128 x 128 bf16]
// * B[smem, 128 rows x D, MN-major].
template <int D>
__device__ __forceinline__ void mma_tmem_by_tile(bool leader, uint32_t d_tmem, uint32_t a_tmem, uint32_t b_smem,
                                                 bool accumulate) {
    using L = Layout<D>;
    constexpr uint32_t idesc = ptx::make_idesc_bf16(kBlock, D, true);
    const uint64_t bd = ptx::make_smem_desc(b_smem, L::kPanelBytes, 1024);
#pragma unroll
    for (int ks = 0; ks < kBlock / 16; ++ks)
        if (leader)
            ptx::mma_ts(d_tmem, a_tmem + ks * 8, bd + ((ks * 16 * 128) >> 4), idesc, (accumulate || ks > 0) ? 1u : 0u);
}

// The dQ kernel's MMA loop, pipelined: as soon as the compute warps have
// read S(j) and dP(j) (sdp_free), S(j+1) and dP(j+1) are issued over them,
// so these products run while dS(j) is computed; dS alternates between two
// TMEM buffers, and dQ += dS(j) K_j follows once dS(j) is in place.  In-order
// execution makes the reuse safe: dQ(j) is issued before S(j+2), so when the
// compute warps see S(j+2) complete, dQ(j) has read dS buffer j & 1.
template <int D>
__device__ void mma_loop_dq(const Common<D>& c, const fa::tc::Sync& sync, uint32_t tmem, int nb) {
    using L = Layout<D>;
    const bool leader = ptx::elect_one();
    auto wait_all = [&](uint32_t bar, uint32_t parity) {
        return __all_sync(0xffffffffu, fa::tc::wait_bar(sync, bar, parity));
    };
    auto commit = [&](uint32_t bar) {
        if (leader) ptx::mma_commit(bar);
    };
    int slot = 0;
    uint32_t phase = 0;
    // the next (K_j, V_j) pair of ring slots
    auto take = [&](int& xs, uint32_t& xp, int& ys, uint32_t& yp) {
        xs = slot;
        ys = slot + 1;
        xp = yp = phase;
        slot = (slot + 2) % kSlots;
        if (slot < 2) phase ^= 1;
    };
    auto issue_sdp = [&](int xs, int ys) {
        mma_rows_by_rows<D>(leader, tmem + L::kTmemS, c.base + L::kAOff, c.slot_addr(xs));   // S = Q K^T
        mma_rows_by_rows<D>(leader, tmem + L::kTmemDP, c.base + L::kBOff, c.slot_addr(ys));  // dP = dO V^T
        commit(c.s_full());
        commit(c.empty(ys));  // V_j is done once dP is
    };
    bool ok = wait_all(c.a_full(), 0) && wait_all(c.b_full(), 0);
    int xs, ys;
    uint32_t xp, yp;
    take(xs, xp, ys, yp);
    ok = ok && wait_all(c.full(xs), xp) && wait_all(c.full(ys), yp);
    if (ok) {
        ptx::tc_fence_after_sync();
        issue_sdp(xs, ys);
    }
    int kslot = xs;
    for (int j = 0; j < nb && ok; ++j) {
        ok = wait_all(c.sdp_free(), j & 1);
        if (!ok) break;
        int next_k = -1;
        if (j + 1 < nb) {
            take(xs, xp, ys, yp);
            ok = wait_all(c.full(xs), xp) && wait_all(c.full(ys), yp);
            if (!ok) break;
            ptx::tc_fence_after_sync();
            issue_sdp(xs, ys);
            next_k = xs;
        }
        ok = wait_all(c.p_full_of(j), (j >> 1) & 1);
        if (!ok) break;
        ptx::tc_fence_after_sync();
        mma_tmem_by_tile<D>(leader, tmem + L::kTmemAcc0, tmem + L::kTmemDS + 64 * (j & 1), c.slot_addr(kslot), j > 0);
        commit(c.empty(kslot));  // K_j is done once dQ(j) is
        kslot = next_k;
    }
    commit(c.done());
    commit(c.drain());
    fa::tc::drain_bar(sync, c.drain(), 0);
    __syncwarp();
}

// The MMA warp's loop, shared by both kernels (A, B resident; streamed pairs
// (X_b, Y_b) in the ring):
//   T0 = A X_b^T   -> kTmemS          T1 = B Y_b^T   -> kTmemDP
//   wait for the compute warps' bf16 results over T0 and T1
//   acc0 += R0 * (dq: X_b | dkdv: Y_b),  acc1 += R1 * X_b (dkdv only)
// where R0 sits over T0 (dS in the dq kernel, P^T in the dK/dV kernel) and
// R1 over T1 (dS^T, dK/dV kernel only).
template <int D, bool kDkdv>
__device__ void mma_loop(const Common<D>& c, const fa::tc::Sync& sync, uint32_t tmem, int nb) {
    using L = Layout<D>;
    const bool leader = ptx::elect_one();
    auto wait_all = [&](uint32_t bar, uint32_t parity) {
        return __all_sync(0xffffffffu, fa::tc::wait_bar(sync, bar, parity));
    };
    auto commit = [&](uint32_t bar) {
        if (leader) ptx::mma_commit(bar);
    };
    bool ok = wait_all(c.a_full(), 0) && wait_all(c.b_full(), 0);
    int slot = 0;
    uint32_t phase = 0;
    for (int b = 0; b < nb && ok; ++b) {
        const int xs = slot, ys = (slot + 1) % kSlots;
        const uint32_t xp = phase, yp = (slot + 1 == kSlots) ? phase ^ 1 : phase;
        slot = (slot + 2) % kSlots;
        if (slot < 2) phase ^= 1;
        ok = wait_all(c.full(xs), xp) && wait_all(c.full(ys), yp);
        if (!ok) break;
        ptx::tc_fence_after_sync();
        mma_rows_by_rows<D>(leader, tmem + L::kTmemS, c.base + L::kAOff, c.slot_addr(xs));
        mma_rows_by_rows<D>(leader, tmem + L::kTmemDP, c.base + L::kBOff, c.slot_addr(ys));
        commit(c.s_full());
        ok = wait_all(c.p_full(), b & 1);
        if (!ok) break;
        ptx::tc_fence_after_sync();
        if (kDkdv) {
            mma_tmem_by_tile<D>(leader, tmem + L::kTmemAcc0, tmem + L::kTmemS, c.slot_addr(ys), b > 0);   // dV += P^T dO
            mma_tmem_by_tile<D>(leader, tmem + L::kTmemAcc1, tmem + L::kTmemDP, c.slot_addr(xs), b > 0);  // dK += dS^T Q
        } else {
            mma_tmem_by_tile<D>(leader, tmem + L::kTmemAcc0, tmem + L::kTmemDS, c.slot_addr(xs), b > 0);  // dQ += dS K
        }
        commit(c.empty(xs));
        commit(c.empty(ys));
    }
    commit(c.done());
    commit(c.drain());
    fa::tc::drain_bar(sync, c.drain(), 0);
    __syncwarp();
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

// ---------------------------------------------------------------- dQ kernel
// CTA = (query block qb, head bh); tiles: Q, dO resident; K_j, V_j streamed.
template <int D, bool kCausal>
__global__ void __launch_bounds__(kThreads, 1)
    fa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                     const Params p) {
    using L = Layout<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = ptx::smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qb = blockIdx.x, bh = blockIdx.y;
    const Common<D> c{base, base + L::kBarOff};
    uint32_t* tmem_base_ptr = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
    const fa::tc::Sync sync{abort_flag, p.status};
    const int nb = kCausal ? min(p.nblocks, qb + 1) : p.nblocks;  // KV blocks this query block uses

    if (threadIdx.x == 0) {
        ptx::mbar_init(c.a_full(), 1);
        ptx::mbar_init(c.b_full(), 1);
        for (int s = 0; s < kSlots; ++s) {
            ptx::mbar_init(c.full(s), 1);
            ptx::mbar_init(c.empty(s), 1);
        }
        ptx::mbar_init(c.s_full(), 1);
        ptx::mbar_init(c.p_full(), 32 * kComputeWarps);
        ptx::mbar_init(c.done(), 1);
        ptx::mbar_init(c.drain(), 1);
        ptx::mbar_init(c.sdp_free(), 32 * kComputeWarps);
        ptx::mbar_init(c.p_full_odd(), 32 * kComputeWarps);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        ptx::tmem_alloc(ptx::smem_addr(tmem_base_ptr), kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    const uint32_t tmem = *tmem_base_ptr;

    if (warp == kLoadWarp) {
        produce<D>(c, sync, &tm_q, &tm_do, qb * kBlock, &tm_k, &tm_v, 0, nb, bh);
    } else if (warp == kMmaWarp) {
        mma_loop_dq<D>(c, sync, tmem, nb);
    } else {
        // one query row per thread (TMEM lane = row within the block); the
        // warp's half h of the key columns
        const int q4 = warp & 3, h = warp >> 2;
        const int r = q4 * 32 + lane;
        const int row = qb * kBlock + r;
        const bool valid = row < p.n;
        const float lse2 = valid ? p.lse[static_cast<int64_t>(bh) * p.n + row] * kLog2e : 0.f;
        const float drow = valid ? p.dsum[static_cast<int64_t>(bh) * p.n + row] : 0.f;
        const uint32_t lane_addr = static_cast<uint32_t>(32 * q4) << 16;
        bool ok = true;
        for (int j = 0; j < nb && ok; ++j) {
            ok = __all_sync(0xffffffffu, fa::tc::wait_bar(sync, c.s_full(), j & 1));
            if (!ok) break;
            ptx::tc_fence_after_sync();
            const uint32_t ds_buf = L::kTmemDS + 64 * (j & 1);
#pragma unroll
            for (int cl = 0; cl < kBlock / 2; cl += 32) {
                const int c0 = h * (kBlock / 2) + cl;
                uint32_t sv[32], gv[32];
                ptx::tmem_ld32_wait(tmem + lane_addr + L::kTmemS + c0, sv);
                ptx::tmem_ld32_wait(tmem + lane_addr + L::kTmemDP + c0, gv);
                if (cl + 32 == kBlock / 2) {
                    // S(j) and dP(j) are in registers: the next pair may overwrite them
                    ptx::tc_fence_before_sync();
                    ptx::mbar_arrive(c.sdp_free());
                }
                uint32_t ds[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    float d2[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int key = j * kBlock + c0 + e + u;
                        const bool use = valid && key < p.n && (!kCausal || key <= row);
                        const float pr = use ? ptx::ex2(__uint_as_float(sv[e + u]) * p.scale_log2 - lse2) : 0.f;
                        d2[u] = pr * (__uint_as_float(gv[e + u]) - drow);
                    }
                    ds[e >> 1] = ptx::pack_bf16x2(d2[0], d2[1]);
                }
                ptx::tmem_st16(tmem + lane_addr + ds_buf + c0 / 2, ds);
            }
            ptx::tmem_st_wait();
            ptx::tc_fence_before_sync();
            ptx::mbar_arrive(c.p_full_of(j));
        }
        if (ok) ok = __all_sync(0xffffffffu, fa::tc::wait_bar(sync, c.done(), 0));
        if (ok) {
            ptx::tc_fence_after_sync();
            store_rows<D>(tmem + lane_addr + L::kTmemAcc0, p.out0 + (static_cast<int64_t>(bh) * p.n + row) * D, valid,
                          p.scale, h * (D / 2));
        }
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    if (warp == kMmaWarp) {
        __syncwarp();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------- dK, dV kernel
// CTA = (key block kb, head bh); tiles: K, V resident; Q_i, dO_i streamed.
template <int D, bool kCausal>
__global__ void __launch_bounds__(kThreads, 1)
    fa_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                       const Params p) {
    using L = Layout<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = ptx::smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kb = blockIdx.x, bh = blockIdx.y;
    const Common<D> c{base, base + L::kBarOff};
    uint32_t* tmem_base_ptr = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
    float* lse2_sm = reinterpret_cast<float*>(smem + L::kVecOff);  // this query block's lse * log2(e)
    float* dsum_sm = lse2_sm + kBlock;                              // and its D
    const fa::tc::Sync sync{abort_flag, p.status};
    const int i_begin = kCausal ? kb : 0;                           // query blocks that see this key block
    const int nb = p.nblocks - i_begin;

    if (threadIdx.x == 0) {
        ptx::mbar_init(c.a_full(), 1);
        ptx::mbar_init(c.b_full(), 1);
        for (int s = 0; s < kSlots; ++s) {
            ptx::mbar_init(c.full(s), 1);
            ptx::mbar_init(c.empty(s), 1);
        }
        ptx::mbar_init(c.s_full(), 1);
        ptx::mbar_init(c.p_full(), 32 * kComputeWarps);
        ptx::mbar_init(c.done(), 1);
        ptx::mbar_init(c.drain(), 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        ptx::tmem_alloc(ptx::smem_addr(tmem_base_ptr), kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    const uint32_t tmem = *tmem_base_ptr;

    if (warp == kLoadWarp) {
        produce<D>(c, sync, &tm_k, &tm_v, kb * kBlock, &tm_q, &tm_do, i_begin, p.nblocks, bh);
    } else if (warp == kMmaWarp) {
        mma_loop<D, true>(c, sync, tmem, nb);
    } else {
        // one key row per thread (TMEM lane = key within the block); the
        // warp's half h of the query columns
        const int q4 = warp & 3, h = warp >> 2;
        const int r = q4 * 32 + lane;
        const int key = kb * kBlock + r;
        const bool kvalid = key < p.n;
        const uint32_t lane_addr = static_cast<uint32_t>(32 * q4) << 16;
        bool ok = true;
        for (int b = 0; b < nb && ok; ++b) {
            const int i = i_begin + b;
            // this query block's statistics, shared by the compute threads
            asm volatile("bar.sync 1, %0;" ::"r"(32 * kComputeWarps) : "memory");
            if (h == 0) {
                const int qrow = i * kBlock + r;
                const bool qv = qrow < p.n;
                lse2_sm[r] = qv ? p.lse[static_cast<int64_t>(bh) * p.n + qrow] * kLog2e : 0.f;
                dsum_sm[r] = qv ? p.dsum[static_cast<int64_t>(bh) * p.n + qrow] : 0.f;
            }
            asm volatile("bar.sync 1, %0;" ::"r"(32 * kComputeWarps) : "memory");
            ok = __all_sync(0xffffffffu, fa::tc::wait_bar(sync, c.s_full(), b & 1));
            if (!ok) break;
            ptx::tc_fence_after_sync();
            uint32_t pp[2][16], ds[2][16];
#pragma unroll
            for (int ci = 0; ci < 2; ++ci) {
                const int c0 = h * (kBlock / 2) + ci * 32;
                uint32_t sv[32], gv[32];
                ptx::tmem_ld32_wait(tmem + lane_addr + L::kTmemS + c0, sv);
                ptx::tmem_ld32_wait(tmem + lane_addr + L::kTmemDP + c0, gv);
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    float p2[2], d2[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int qc = c0 + e + u;  // query within the block
                        const int qrow = i * kBlock + qc;
                        const bool use = kvalid && qrow < p.n && (!kCausal || key <= qrow);
                        p2[u] = use ? ptx::ex2(__uint_as_float(sv[e + u]) * p.scale_log2 - lse2_sm[qc]) : 0.f;
                        d2[u] = p2[u] * (__uint_as_float(gv[e + u]) - dsum_sm[qc]);
                    }
                    pp[ci][e >> 1] = ptx::pack_bf16x2(p2[0], p2[1]);
                    ds[ci][e >> 1] = ptx::pack_bf16x2(d2[0], d2[1]);
                }
            }
            // P^T goes over S^T and dS^T over dP^T: the second warp's results
            // land on columns the first warp reads, so the pair meets first
            asm volatile("bar.sync %0, 64;" ::"r"(2 + q4) : "memory");
#pragma unroll
            for (int ci = 0; ci < 2; ++ci) {
                const int c0 = h * (kBlock / 2) + ci * 32;
                ptx::tmem_st16(tmem + lane_addr + L::kTmemS + c0 / 2, pp[ci]);
                ptx::tmem_st16(tmem + lane_addr + L::kTmemDP + c0 / 2, ds[ci]);
            }
            ptx::tmem_st_wait();
            ptx::tc_fence_before_sync();
            ptx::mbar_arrive(c.p_full());
        }
        if (ok) ok = __all_sync(0xffffffffu, fa::tc::wait_bar(sync, c.done(), 0));
        if (ok) {
            ptx::tc_fence_after_sync();
            const int64_t off = (static_cast<int64_t>(bh) * p.n + key) * D;
            store_rows<D>(tmem + lane_addr + L::kTmemAcc0, p.out0 + off, kvalid, 1.f, h * (D / 2));      // dV
            store_rows<D>(tmem + lane_addr + L::kTmemAcc1, p.out1 + off, kvalid, p.scale, h * (D / 2));  // dK
        }
    }
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
