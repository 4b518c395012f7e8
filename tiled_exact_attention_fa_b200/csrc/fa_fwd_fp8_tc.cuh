// fa_fwd_fp8_tc.cuh -- attention forward with 8-bit float (E4M3) inputs on the
// sm_100a tensor cores.
//
// What it computes (per head): the attention of fa_fwd_tc.cuh,
//   O = softmax(scale * (dq Q8)(dk K8)^T [causal]) (dv V8),  lse per row,
// where Q8, K8, V8 hold OCP E4M3 values and dq, dk, dv are per-tensor factors
// (the usual way 8-bit tensors carry their range).  The pages name low
// precision (FP8) as the third generation's step on Hopper (Chapter 15 --
// FlashAttention, "FlashAttention Evolution", FA-3) without fixing its
// arithmetic; the reading here: Q K^T and P V run on the tensor core in E4M3
// with fp32 accumulation, P is rounded to E4M3 (round to nearest, saturating)
// only as the operand of P V, the running max and sum stay fp32, and O is
// written in bf16.  dq dk fold into the exponent's scale, dv into the final
// normalisation, so the kernel never rescales an input.
//
// Same roles as the bf16 kernel (persistent CTAs, a producer warp, one
// MMA-issuing warp, sixteen softmax warps over two 128-row query tiles), with
// what 8-bit operands change:
//   * a 128 x 128 tile is one 128-byte swizzle panel (16 KB);
//   * tcgen05.mma kind::f8f6f4 consumes 32 elements of the reduction per
//     instruction: S = Q K^T is 4 MMAs and O += P V is 4 MMAs per block, half
//     the tensor-core time of bf16, which leaves the softmax as the bound;
//   * so the softmax must never wait for the tensor core.  P (16 KB per tile
//     in E4M3) goes to a double-buffered shared-memory tile instead of over S
//     in TMEM, and a warp signals "S consumed" as soon as its scores are in
//     registers: the MMA warp then computes the next block's S while this
//     block is exponentiated, and P V runs behind, off the softmax's path;
//   * the softmax warps read S with the .16x32bx2 TMEM shape: thread t of a
//     warp owns one row (lane t % 16 of the warp's 16 lanes) and 64
//     consecutive keys (half t / 16 of the block).  Row reductions finish
//     with one shuffle (lanes t and t ^ 16 share a row), and the thread's 64
//     P bytes are four 16-byte chunks of the row of the K-major, 128-byte
//     swizzled A operand;
//   * P is rounded to E4M3, whose largest finite value is 448.  Every block's
//     exact max is taken, but the running max m only moves to it when it
//     exceeds m by more than 8 (log2 units): p = 2^(s - m) <= 2^8 = 256, so
//     nothing saturates, and O and l are rescaled only on such rare jumps.
//
// Shared memory: Q (2 x 16 KB), a ring of 8 K/V slots (16 KB each), P (2 tiles
// x 2 buffers x 16 KB).  TMEM columns (512): S_0 at 0, S_1 at 128, O_0 at 256,
// O_1 at 384.  Head dim 128 only.
//
// Every mbarrier wait is bounded (tc::wait_bar / tc::drain_bar); on expiry the
// CTA records the timeout in the device status word, leaves its loops, drains
// its copies and MMAs and frees TMEM.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "fa_fwd_tc.cuh"
#include "sm100_ptx.cuh"

namespace fa {
namespace tc8 {

using tc::kBlockM;
using tc::kBlockN;
using tc::kSchedDepth;
using tc::kTmemCols;
using tc::kUnitRows;

constexpr int kSoftmaxWarps = 16;      // 8 per query tile
constexpr int kMmaWarp = 16;
constexpr int kLoadWarp = 17;
constexpr int kThreads = 576;

constexpr int D = 128;                 // head dim (one 128-byte row of E4M3)
constexpr int kSlots = 8;              // K/V ring slots
constexpr float kMaxSlack = 8.0f;      // log2 units a block's max may exceed the running max by

struct Layout {
    static constexpr int kTileBytes = kBlockM * D;  // 128 rows x 128 one-byte elements
    static constexpr int kQOff = 0;
    static constexpr int kRingOff = kQOff + 2 * kTileBytes;
    static constexpr int kPOff = kRingOff + kSlots * kTileBytes;  // P[tile][buffer]
    static constexpr int kBarOff = kPOff + 4 * kTileBytes;
    // mbarrier indices: q_full[2], q_empty[2], kv_full[S], kv_empty[S], s_full[2], s_free[2],
    // p_full[2][2], p_free[2][2], o_full[2], sched_full[kSchedDepth], sched_empty[kSchedDepth], drain
    static constexpr int kBarQFull = 0, kBarQEmpty = 2, kBarKvFull = 4, kBarKvEmpty = 4 + kSlots;
    static constexpr int kBarSFull = 4 + 2 * kSlots, kBarSFree = kBarSFull + 2, kBarPFull = kBarSFree + 2;
    static constexpr int kBarPFree = kBarPFull + 4, kBarOFull = kBarPFree + 4, kBarSchedFull = kBarOFull + 2;
    static constexpr int kBarSchedEmpty = kBarSchedFull + kSchedDepth, kBarDrain = kBarSchedEmpty + kSchedDepth;
    static constexpr int kNumBars = kBarDrain + 1;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;  // tmem base, abort flag, unit ring
    static constexpr int kClockOff = (kMiscOff + 8 + 4 * kSchedDepth + 7) & ~7;  // int64[2]: start clock, timer
    static constexpr int kBytes = kClockOff + 16;
    static constexpr int kSmemBytes = kBytes + 1024;         // slack for 1024-byte alignment
    static constexpr uint32_t kTmemS = 0;
    static constexpr uint32_t kTmemO = 256;
    static_assert(kSmemBytes <= 232448, "shared memory per block");
};

struct Params {
    tc::Params base;   // o (bf16), lse, status, queue, sizes; scale_log2 = scale * dq * dk * log2(e)
    float o_scale;     // dv: the factor of V, applied with 1/l
};

// ----------------------------------------------------------------- instructions
// Wrappers written from the PTX ISA's descriptions of tcgen05.mma (kind::f8f6f4),
// the .16x32bx2 tcgen05.ld/st shape and cvt to e4m3x2.

// Instruction descriptor for kind::f8f6f4 with E4M3 A and B and fp32 D:
//   [4,6) D format (1 = f32), [7,10) A format (0 = E4M3), [10,13) B format (0 = E4M3),
//   [15] A major (0 = K), [16] B major (0 = K, 1 = MN), [17,23) N >> 3, [24,29) M >> 4.
__host__ __device__ constexpr uint32_t make_idesc_e4m3(int M, int N, bool b_mn_major) {
    return (1u << 4) | ((b_mn_major ? 1u : 0u) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(M >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem]^T, 8-bit float operands.
__device__ __forceinline__ void mma_ss_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem], A (four 8-bit values per column) read from tensor memory.
__device__ __forceinline__ void mma_ts_f8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// .16x32bx2 shape: a warp accesses 16 TMEM lanes starting at the lane field of
// taddr; thread t reads/writes lane t % 16, columns [col + kSplit * (t / 16),
// + num) with num = the register count.
#define FA_R8(b) "=r"(r[b + 0]), "=r"(r[b + 1]), "=r"(r[b + 2]), "=r"(r[b + 3]), \
                 "=r"(r[b + 4]), "=r"(r[b + 5]), "=r"(r[b + 6]), "=r"(r[b + 7])
#define FA_W8(b) "r"(r[b + 0]), "r"(r[b + 1]), "r"(r[b + 2]), "r"(r[b + 3]), \
                 "r"(r[b + 4]), "r"(r[b + 5]), "r"(r[b + 6]), "r"(r[b + 7])

template <int kSplit>
__device__ __forceinline__ void tmem_ld16x32bx2_x64_wait(uint32_t taddr, uint32_t (&r)[64]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x32bx2.x64.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, "
        "%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, "
        "%48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64], %65;\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : FA_R8(0), FA_R8(8), FA_R8(16), FA_R8(24), FA_R8(32), FA_R8(40), FA_R8(48), FA_R8(56)
        : "r"(taddr), "n"(kSplit)
        : "memory");
}
template <int kSplit>
__device__ __forceinline__ void tmem_ld16x32bx2_x32_wait(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32], %33;\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : FA_R8(0), FA_R8(8), FA_R8(16), FA_R8(24)
        : "r"(taddr), "n"(kSplit)
        : "memory");
}
template <int kSplit>
__device__ __forceinline__ void tmem_ld16x32bx2_x16_wait(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x32bx2.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16], %17;\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : FA_R8(0), FA_R8(8)
        : "r"(taddr), "n"(kSplit)
        : "memory");
}
template <int kSplit>
__device__ __forceinline__ void tmem_st16x32bx2_x16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.16x32bx2.x16.b32 [%0], %1, "
        "{%2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17};" ::"r"(taddr),
        "n"(kSplit), FA_W8(0), FA_W8(8)
        : "memory");
}
#undef FA_R8
#undef FA_W8

// Four floats to four E4M3 bytes (round to nearest even, saturating to +-448):
// x0 in bits [0,8), x1 in [8,16), x2 in [16,24), x3 in [24,32).
__device__ __forceinline__ uint32_t pack_e4m3x4(float x0, float x1, float x2, float x3) {
    uint32_t r;
    asm("{\n\t.reg .b16 lo, hi;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n\t"
        "mov.b32 %0, {lo, hi};\n\t}"
        : "=r"(r)
        : "f"(x0), "f"(x1), "f"(x2), "f"(x3));
    return r;
}

// Make this thread's shared-memory writes visible to the tensor core (async proxy).
__device__ __forceinline__ void fence_async_shared() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ----------------------------------------------------------------- kernel

template <bool kCausal>
__global__ void __launch_bounds__(kThreads, 1)
    fa_fwd_e4m3_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const Params prm) {
    using L = Layout;
    const tc::Params& p = prm.base;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = ptx::smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    const uint32_t bar0 = base + L::kBarOff;
    auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
    auto q_full = [&](int t) { return bar(L::kBarQFull + t); };
    auto q_empty = [&](int t) { return bar(L::kBarQEmpty + t); };
    auto kv_full = [&](int s) { return bar(L::kBarKvFull + s); };
    auto kv_empty = [&](int s) { return bar(L::kBarKvEmpty + s); };
    auto s_full = [&](int t) { return bar(L::kBarSFull + t); };
    auto s_free = [&](int t) { return bar(L::kBarSFree + t); };
    // P_t of block k is announced on p_full(t, k & 1): with the next S issued
    // early, a tile's softmax can finish block k + 1 before the MMA warp has
    // seen block k, so one barrier could complete two phases unobserved.
    auto p_full = [&](int t, int b) { return bar(L::kBarPFull + 2 * t + b); };
    auto p_free = [&](int t, int b) { return bar(L::kBarPFree + 2 * t + b); };
    auto o_full = [&](int t) { return bar(L::kBarOFull + t); };
    auto sched_full = [&](int i) { return bar(L::kBarSchedFull + i); };
    auto sched_empty = [&](int i) { return bar(L::kBarSchedEmpty + i); };
    const uint32_t drain = bar(L::kBarDrain);

    uint32_t* tmem_base_ptr = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
    volatile int* unit_ring = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 8);
    const tc::Sync sync{abort_flag, p.status};

    if (threadIdx.x == 0) {
        for (int t = 0; t < 2; ++t) {
            ptx::mbar_init(q_full(t), 1);
            ptx::mbar_init(q_empty(t), 1);
            ptx::mbar_init(s_full(t), 1);
            ptx::mbar_init(s_free(t), 32 * (kSoftmaxWarps / 2));
            ptx::mbar_init(p_full(t, 0), 32 * (kSoftmaxWarps / 2));
            ptx::mbar_init(p_full(t, 1), 32 * (kSoftmaxWarps / 2));
            ptx::mbar_init(p_free(t, 0), 1);
            ptx::mbar_init(p_free(t, 1), 1);
            ptx::mbar_init(o_full(t), 1);
        }
        for (int s = 0; s < kSlots; ++s) {
            ptx::mbar_init(kv_full(s), 1);
            ptx::mbar_init(kv_empty(s), 1);
        }
        for (int i = 0; i < kSchedDepth; ++i) {
            ptx::mbar_init(sched_full(i), 1);
            ptx::mbar_init(sched_empty(i), 1 + kSoftmaxWarps);
        }
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
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    tc::grid_dependency_wait();
    const uint32_t tmem = *tmem_base_ptr;

    if (warp == kLoadWarp) {
        tc::clock_start(p, smem + L::kClockOff, lane == 0);
        // ------------------------------------------------------------ producer
        const bool leader = ptx::elect_one();
        const uint64_t keep = ptx::policy_evict_last();   // K/V: re-read by the head's other units
        const uint64_t once = ptx::policy_evict_first();  // Q: read once
        int slot = 0;
        uint32_t phase = 0, nloads = 0;
        uint32_t q_issued[2] = {0, 0};
        bool ok = true;
        for (uint32_t it = 0; ok; ++it) {
            const int rs = it % kSchedDepth;
            ok = __all_sync(0xffffffffu, tc::wait_bar(sync, sched_empty(rs), ((it / kSchedDepth) & 1) ^ 1));
            if (!ok) break;
            int u = 0;
            if (leader) {
                u = static_cast<int>(atomicAdd(p.sched, 1u));
                if (u >= p.num_units) u = -1;
                unit_ring[rs] = u;
                ptx::mbar_arrive(sched_full(rs));
            }
            u = __shfl_sync(0xffffffffu, u, __ffs(__ballot_sync(0xffffffffu, leader)) - 1);
            if (u < 0) {
                tc::launch_dependents();
                break;
            }

            const tc::Unit w = tc::decode_unit(u, p, kCausal);
            const int n1 = tc::num_kv_blocks(p, w.qb, 1, kCausal);
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                if (!ok) break;
                ok = __all_sync(0xffffffffu, tc::wait_bar(sync, q_empty(t), (it & 1) ^ 1));
                if (!ok) break;
                q_issued[t] = (it & 1) + 1;
                if (leader) {
                    ptx::mbar_arrive_expect_tx(q_full(t), L::kTileBytes);
                    ptx::tma_load_3d(base + L::kQOff + t * L::kTileBytes, &tm_q, q_full(t), 0,
                                     w.qb * kUnitRows + t * kBlockM, w.bh, once);
                }
            }
            for (int j = 0; j < n1 && ok; ++j) {
                for (int kv = 0; kv < 2 && ok; ++kv) {
                    ok = __all_sync(0xffffffffu, tc::wait_bar(sync, kv_empty(slot), phase ^ 1));
                    if (!ok) break;
                    if (leader) {
                        ptx::mbar_arrive_expect_tx(kv_full(slot), L::kTileBytes);
                        ptx::tma_load_3d(base + L::kRingOff + slot * L::kTileBytes, kv == 0 ? &tm_k : &tm_v,
                                         kv_full(slot), 0, j * kBlockN, w.bh, keep);
                    }
                    ++nloads;
                    if (++slot == kSlots) {
                        slot = 0;
                        phase ^= 1;
                    }
                }
            }
        }
        // Drain: every issued copy lands before shared memory is released.
        for (uint32_t s = 0; s < static_cast<uint32_t>(kSlots) && s < nloads; ++s) {
            const uint32_t last = s + kSlots * ((nloads - 1 - s) / kSlots);
            tc::drain_bar(sync, kv_full(s), (last / kSlots) & 1);
        }
        for (int t = 0; t < 2; ++t)
            if (q_issued[t]) tc::drain_bar(sync, q_full(t), q_issued[t] - 1);
        if (leader) {
            __threadfence();
            if (atomicAdd(p.sched + 1, 1u) == gridDim.x - 1) {
                atomicExch(p.sched, 0u);
                atomicExch(p.sched + 1, 0u);
            }
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        // The whole warp runs the loop (warp-uniform descriptors and waits);
        // one elected lane issues every MMA and commit.  Per block j and tile
        // t: S_t(j+1) as soon as the softmax has read S_t(j), then P_t(j) V_j
        // as soon as P_t(j) is in shared memory.
        const bool leader = ptx::elect_one();
        constexpr uint32_t idesc_s = make_idesc_e4m3(kBlockM, kBlockN, false);
        constexpr uint32_t idesc_o = make_idesc_e4m3(kBlockM, D, true);
        const uint64_t desc_q0 = ptx::make_smem_desc(base + L::kQOff, 16, 1024);
        const uint64_t desc_k0 = ptx::make_smem_desc(base + L::kRingOff, 16, 1024);
        const uint64_t desc_v0 = ptx::make_smem_desc(base + L::kRingOff, L::kTileBytes, 1024);
        const uint64_t desc_p0 = ptx::make_smem_desc(base + L::kPOff, 16, 1024);
        int slot = 0;
        uint32_t phase = 0;
        uint32_t sf_phase[2] = {0, 0};
        uint32_t pv_count[2] = {0, 0};  // P V products issued per tile (selects the P buffer)
        bool ok = true;

        // S_t = Q_t K^T: 4 MMAs of 32 elements (32 bytes along the swizzled row).
        auto issue_s = [&](int t, int kslot) {
            const uint64_t qd = desc_q0 + ((t * L::kTileBytes) >> 4);
            const uint64_t kd = desc_k0 + ((kslot * L::kTileBytes) >> 4);
#pragma unroll
            for (int ks = 0; ks < D / 32; ++ks)
                if (leader) mma_ss_f8(tmem + L::kTmemS + t * kBlockN, qd + 2 * ks, kd + 2 * ks, idesc_s, ks > 0);
        };
        // O_t (+)= P_t V: 4 MMAs of 32 keys; P from its shared-memory buffer
        // (K-major like Q), V as an MN-major operand (32 rows of 128 bytes per step).
        auto issue_pv = [&](int t, int vslot, bool accumulate) {
            const int b = static_cast<int>(pv_count[t] & 1u);
            const uint64_t pd = desc_p0 + (((2 * t + b) * L::kTileBytes) >> 4);
            const uint64_t vd = desc_v0 + ((vslot * L::kTileBytes) >> 4);
#pragma unroll
            for (int ks = 0; ks < kBlockN / 32; ++ks)
                if (leader)
                    mma_ss_f8(tmem + L::kTmemO + t * D, pd + 2 * ks, vd + ((ks * 32 * 128) >> 4), idesc_o,
                              (accumulate || ks > 0) ? 1u : 0u);
            if (leader) ptx::mma_commit(p_free(t, b));  // the buffer may be rewritten once these complete
            ++pv_count[t];
        };
        auto commit = [&](uint32_t bar) {
            if (leader) ptx::mma_commit(bar);
        };
        auto next_slot = [&](int& s, uint32_t& ph) {
            s = slot;
            ph = phase;
            if (++slot == kSlots) {
                slot = 0;
                phase ^= 1;
            }
        };
        auto wait_all = [&](uint32_t bar, uint32_t parity) {
            return __all_sync(0xffffffffu, tc::wait_bar(sync, bar, parity));
        };

        for (uint32_t it = 0; ok; ++it) {
            const int rs = it % kSchedDepth;
            ok = wait_all(sched_full(rs), (it / kSchedDepth) & 1);
            if (!ok) break;
            const int u = unit_ring[rs];
            __syncwarp();
            if (leader) ptx::mbar_arrive(sched_empty(rs));
            if (u < 0) break;

            const tc::Unit w = tc::decode_unit(u, p, kCausal);
            const int n0 = tc::num_kv_blocks(p, w.qb, 0, kCausal);
            const int n1 = tc::num_kv_blocks(p, w.qb, 1, kCausal);
            ok = wait_all(q_full(0), it & 1) && wait_all(q_full(1), it & 1);
            if (!ok) break;
            int sk, sv;
            uint32_t pk, pv;
            next_slot(sk, pk);
            ok = wait_all(kv_full(sk), pk);
            if (!ok) break;
            ptx::tc_fence_after_sync();
            issue_s(0, sk);
            commit(s_full(0));
            if (n0 == 1) commit(q_empty(0));
            issue_s(1, sk);
            commit(s_full(1));
            if (n1 == 1) commit(q_empty(1));
            commit(kv_empty(sk));

            for (int j = 0; j < n1 && ok; ++j) {
                const bool more0 = j + 1 < n0, more1 = j + 1 < n1;
                next_slot(sv, pv);  // V_j (loaded before K_{j+1})
                if (more1) {
                    next_slot(sk, pk);
                    ok = wait_all(kv_full(sk), pk);
                    if (!ok) break;
                }
                if (more0) {
                    ok = wait_all(s_free(0), sf_phase[0]);
                    if (!ok) break;
                    sf_phase[0] ^= 1;
                    ptx::tc_fence_after_sync();
                    issue_s(0, sk);
                    commit(s_full(0));
                    if (j + 1 == n0 - 1) commit(q_empty(0));
                }
                if (more1) {
                    ok = wait_all(s_free(1), sf_phase[1]);
                    if (!ok) break;
                    sf_phase[1] ^= 1;
                    ptx::tc_fence_after_sync();
                    issue_s(1, sk);
                    commit(s_full(1));
                    if (j + 1 == n1 - 1) commit(q_empty(1));
                    commit(kv_empty(sk));
                }
                ok = wait_all(kv_full(sv), pv);
                if (!ok) break;
                if (j < n0) {
                    ok = wait_all(p_full(0, pv_count[0] & 1u), (pv_count[0] >> 1) & 1u);
                    if (!ok) break;
                    ptx::tc_fence_after_sync();
                    issue_pv(0, sv, j > 0);
                    if (j == n0 - 1) commit(o_full(0));
                }
                ok = wait_all(p_full(1, pv_count[1] & 1u), (pv_count[1] >> 1) & 1u);
                if (!ok) break;
                ptx::tc_fence_after_sync();
                issue_pv(1, sv, j > 0);
                if (j == n1 - 1) commit(o_full(1));
                commit(kv_empty(sv));
            }
        }
        commit(drain);
        tc::drain_bar(sync, drain, 0);
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax warps
        // Warps 0-7 serve query tile 0 and warps 8-15 tile 1; the two warps of
        // a tile that share TMEM lane quarter q (= warp % 4) take its 16-lane
        // halves h.  Thread `lane` owns row rr (lane % 16 of the half) and
        // keys [64 c2, 64 c2 + 64) of every block, c2 = lane / 16.
        const int t = warp >> 3;
        const int q = warp & 3;
        const int h = (warp >> 2) & 1;
        const int c2 = lane >> 4;
        const int rr = 32 * q + 16 * h + (lane & 15);
        const uint32_t lane_addr = static_cast<uint32_t>(32 * q + 16 * h) << 16;
        const uint32_t tmem_s = tmem + lane_addr + L::kTmemS + t * kBlockN;
        const uint32_t tmem_o = tmem + lane_addr + L::kTmemO + t * D;
        // This thread's 64 bytes of a P row: chunks 4 c2 .. 4 c2 + 3 (16 bytes
        // each) of row rr, placed by the 128-byte swizzle (chunk ^ row % 8).
        uint8_t* p_row = smem + L::kPOff + t * 2 * L::kTileBytes + (rr >> 3) * 1024 + (rr & 7) * 128;
        const float sl = p.scale_log2;
        uint32_t s_phase = 0, o_phase = 0;
        uint32_t blk = 0;  // blocks this thread has processed (P buffer blk & 1)
        bool ok = true;

        for (uint32_t it = 0; ok; ++it) {
            const int rs = it % kSchedDepth;
            ok = __all_sync(0xffffffffu, tc::wait_bar(sync, sched_full(rs), (it / kSchedDepth) & 1));
            if (!ok) break;
            const int u = unit_ring[rs];
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(sched_empty(rs));
            if (u < 0) break;

            const tc::Unit w = tc::decode_unit(u, p, kCausal);
            const int nt = tc::num_kv_blocks(p, w.qb, t, kCausal);
            const int tile_row0 = w.qb * kUnitRows + t * kBlockM;
            const int row = tile_row0 + rr;
            float m_run = -INFINITY;  // running max of the row, log2 units
            float l_run = 0.f;        // this thread's share of the row sum

            for (int j = 0; j < nt; ++j, ++blk) {
                ok = __all_sync(0xffffffffu, tc::wait_bar(sync, s_full(t), s_phase));
                if (!ok) break;
                s_phase ^= 1;
                ptx::tc_fence_after_sync();

                const int key0 = j * kBlockN + 64 * c2;  // first key of this thread
                const bool need_mask =
                    (j * kBlockN + kBlockN > p.n) || (kCausal && j * kBlockN + kBlockN - 1 > tile_row0);
                const float slv = need_mask ? 1.f : sl;  // masked blocks are pre-scaled
                uint32_t sr[64];
                float(&s)[64] = *reinterpret_cast<float(*)[64]>(sr);
                tmem_ld16x32bx2_x64_wait<64>(tmem_s, sr);
                // S_t is in registers: the tensor core may overwrite it with
                // the next block's scores while this one is exponentiated.
                if (j + 1 < nt) {
                    ptx::tc_fence_before_sync();
                    ptx::mbar_arrive(s_free(t));
                }
                if (need_mask) {
                    const int lim = kCausal ? min(p.n - 1, row) : (p.n - 1);
#pragma unroll
                    for (int i = 0; i < 64; ++i) s[i] = (key0 + i <= lim) ? s[i] * sl : -INFINITY;
                }
                // Exact row max in log2 units (both halves of the row): four
                // running extremes over s[0..59] in steps of eight, then s[60..63].
                auto block_max = [&]() {
                    float e0 = s[0], e1 = s[1], e2 = s[2], e3 = s[3];
                    if (slv >= 0.f) {
#pragma unroll
                        for (int i = 4; i < 60; i += 8) {
                            e0 = ptx::max3(e0, s[i], s[i + 1]);
                            e1 = ptx::max3(e1, s[i + 2], s[i + 3]);
                            e2 = ptx::max3(e2, s[i + 4], s[i + 5]);
                            e3 = ptx::max3(e3, s[i + 6], s[i + 7]);
                        }
                        e0 = ptx::max3(e0, s[60], s[61]);
                        e1 = ptx::max3(e1, s[62], s[63]);
                        float mx = fmaxf(fmaxf(e0, e1), fmaxf(e2, e3));
                        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                        return mx * slv;
                    }
#pragma unroll
                    for (int i = 4; i < 60; i += 8) {
                        e0 = ptx::min3(e0, s[i], s[i + 1]);
                        e1 = ptx::min3(e1, s[i + 2], s[i + 3]);
                        e2 = ptx::min3(e2, s[i + 4], s[i + 5]);
                        e3 = ptx::min3(e3, s[i + 6], s[i + 7]);
                    }
                    e0 = ptx::min3(e0, s[60], s[61]);
                    e1 = ptx::min3(e1, s[62], s[63]);
                    float mn = fminf(fminf(e0, e1), fminf(e2, e3));
                    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 16));
                    return mn * slv;
                };
                // p = 2^(s * slv - m), packed four keys per 32-bit word (the
                // first key in the low byte) and written as four 16-byte
                // chunks of the row to P buffer `prow`; a0 + a1 is this
                // thread's share of the row sum over the unrounded values.
                float a0, a1;
                auto exponentiate = [&](float neg_m, uint8_t* prow) {
                    a0 = a1 = 0.f;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t wd[4];
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const int i = 4 * c + k;
                            float x0, x1, x2, x3;
                            ptx::fma2(x0, x1, s[4 * i], s[4 * i + 1], slv, slv, neg_m, neg_m);
                            ptx::fma2(x2, x3, s[4 * i + 2], s[4 * i + 3], slv, slv, neg_m, neg_m);
                            const float p0 = ptx::ex2(x0), p1 = ptx::ex2(x1);
                            const float p2 = ptx::ex2(x2), p3 = ptx::ex2(x3);
                            wd[k] = pack_e4m3x4(p0, p1, p2, p3);
                            ptx::add2(a0, a1, a0, a1, p0, p1);
                            ptx::add2(a0, a1, a0, a1, p2, p3);
                        }
                        const int chunk = (4 * c2 + c) ^ (rr & 7);
                        *reinterpret_cast<uint4*>(prow + 16 * chunk) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
                    }
                };
                auto neg_of = [](float m) { return (m == -INFINITY) ? 0.f : -m; };

                // Online softmax with a lazily moved running max (see the file
                // header): m moves to the block's max only when that exceeds
                // it by more than kMaxSlack, so every p stays <= 2^kMaxSlack.
                float alpha = 1.f;
                bool rescale_o = false;
                const float mx = block_max();
                if (j == 0) {
                    m_run = mx;
                } else if (mx > m_run + kMaxSlack) {
                    alpha = ptx::ex2(m_run - mx);
                    m_run = mx;
                    rescale_o = true;
                }
                // P_t(j) goes to buffer blk & 1 once the P V that read it two
                // blocks ago is complete.
                const int b = static_cast<int>(blk & 1u);
                if (blk >= 2) {
                    ok = __all_sync(0xffffffffu, tc::wait_bar(sync, p_free(t, b), ((blk >> 1) - 1) & 1u));
                    if (!ok) break;
                }
                exponentiate(neg_of(m_run), p_row + b * L::kTileBytes);
                l_run = l_run * alpha + (a0 + a1);

                // Rescale this row of O_t once P_t(j-1) V is complete (both
                // halves of the row agree on alpha).
                if (__any_sync(0xffffffffu, rescale_o)) {
                    const uint32_t prev = blk - 1;
                    ok = __all_sync(0xffffffffu,
                                    tc::wait_bar(sync, p_free(t, static_cast<int>(prev & 1u)), (prev >> 1) & 1u));
                    if (!ok) break;
                    ptx::tc_fence_after_sync();
#pragma unroll
                    for (int c0 = 0; c0 < D / 2; c0 += 16) {
                        uint32_t ov[16];
                        tmem_ld16x32bx2_x16_wait<64>(tmem_o + c0, ov);
#pragma unroll
                        for (int i = 0; i < 16; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
                        tmem_st16x32bx2_x16<64>(tmem_o + c0, ov);
                    }
                    ptx::tmem_st_wait();
                }
                fence_async_shared();
                ptx::tc_fence_before_sync();
                ptx::mbar_arrive(p_full(t, b));
            }
            if (!ok) break;

            // Epilogue: the row sum is complete once the two halves are added.
            l_run += __shfl_xor_sync(0xffffffffu, l_run, 16);
            ok = __all_sync(0xffffffffu, tc::wait_bar(sync, o_full(t), o_phase));
            if (!ok) break;
            o_phase ^= 1;
            ptx::tc_fence_after_sync();
            const bool valid = row < p.n;
            if (c2 == 0 && valid) {
                const float mu = (m_run == -INFINITY) ? 0.f : m_run;
                p.lse[static_cast<int64_t>(w.bh) * p.n + row] = (mu + log2f(l_run)) * 0.69314718055994531f;
            }
            // O = dv * O_acc / l in bf16, written once: this thread's 64 columns of its row.
            const float inv_l = prm.o_scale / l_run;
            __nv_bfloat16* orow_g = p.o + (static_cast<int64_t>(w.bh) * p.n + row) * D + 64 * c2;
#pragma unroll
            for (int c0 = 0; c0 < D / 2; c0 += 32) {
                uint32_t acc[32];
                tmem_ld16x32bx2_x32_wait<64>(tmem_o + c0, acc);
                uint32_t packed[16];
#pragma unroll
                for (int c = 0; c < 32; c += 2)
                    packed[c >> 1] = ptx::pack_bf16x2(__uint_as_float(acc[c]) * inv_l,
                                                      __uint_as_float(acc[c + 1]) * inv_l);
                if (valid) {
                    uint4* dst = reinterpret_cast<uint4*>(orow_g + c0);
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
                }
            }
            ptx::tc_fence_before_sync();
        }
    }

    // ---------------------------------------------------------------- teardown
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    if (warp == kMmaWarp) {
        __syncwarp();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
    tc::clock_end(p, smem + L::kClockOff);
}

}  // namespace tc8
}  // namespace fa
