// fa_fwd_tc1.cuh -- bf16 attention forward for problems too small to fill
// the GPU with 256-row units: one 128-row query tile per work unit, so twice
// as many units (CTAs) as the two-tile kernel of fa_fwd_tc.cuh, with the
// score tile double-buffered in tensor memory.
//
// Same computation as fa_fwd_tc.cuh ("FlashAttention: Tiled & Fused", the
// tiled forward; "FlashAttention, Playable", EP 04, the online softmax with
// its rescale), the same reading of the running max (exact on a unit's first
// block, then kept while no thread's share of a row sum exceeds
// kStaleMaxBound) and the same two row sums (fp32 for lse, bf16-consistent
// for O), so the two kernels give bit-identical results.  What differs:
//   * warps 0-7 (two per TMEM lane quarter, 16 rows each) own the one tile;
//     warp 8 issues the MMAs, warp 9 loads Q, K and V with TMA;
//   * TMEM: S in two 128-column buffers (S_j in buffer j & 1, P_j written
//     over its first 64 columns), O in columns 256..256+D.  The MMA warp
//     issues S_{j+2} right after P_j V_j, so the softmax warps find the next
//     block's scores ready and only wait for P_{j-1} V before touching O;
//   * each warp stores its rows of O straight from registers at the end of a
//     unit (small problems: no staging tile, no TMA store).
// The host picks this kernel when a simulation of both kernels' schedules
// says it finishes first: small problems (every 128-row tile on its own SM)
// and medium causal ones, where the two-tile kernel's heaviest 256-row unit
// would set the launch's length.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "fa_fwd_tc.cuh"
#include "sm100_ptx.cuh"

namespace fa {
namespace tc1 {

using tc::kBlockM;
using tc::kBlockN;
using tc::kSchedDepth;
using tc::kStaleMaxBound;
using tc::kTmemCols;
using tc::Params;
using tc::Sync;
using tc::Unit;

constexpr int kSoftmaxWarps = 8;   // two per TMEM lane quarter, 16 rows each
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp = 9;
constexpr int kThreads = 320;

template <int D>
struct Layout {
    static_assert(D == 64 || D == 128, "head dim");
    static constexpr int kHalves = D / 64;
    static constexpr int kPanelBytes = kBlockM * 128;
    static constexpr int kTileBytes = kPanelBytes * kHalves;
    static constexpr int kSlots = (D == 128) ? 4 : 8;
    static constexpr int kQOff = 0;                                // two Q buffers (alternate units)
    static constexpr int kRingOff = kQOff + 2 * kTileBytes;
    static constexpr int kBarOff = kRingOff + kSlots * kTileBytes;
    // q_full[2], q_empty[2], kv_full[S], kv_empty[S], s_full[2], p_full[2], pv_done, o_free,
    // sched_full[kSchedDepth], sched_empty[kSchedDepth], drain, pair[4]
    static constexpr int kNumBars = 2 + 2 + 2 * kSlots + 2 + 4 + 2 * kSchedDepth + 1 + 4;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kInvLOff = (kMiscOff + 8 + 4 * kSchedDepth + 15) & ~15;  // float[2 units][128]
    static constexpr int kClockOff = kInvLOff + 2 * kBlockM * 4;  // int64[2]: start clock, timer
    static constexpr int kBytes = kClockOff + 16;
    static constexpr int kSmemBytes = kBytes + 1024;
    static constexpr uint32_t kTmemS = 0;      // S buffers at 0 and 128; P over the first 64 columns of each
    static constexpr uint32_t kTmemO = 256;
    static_assert(kSmemBytes <= 232448, "shared memory");
};

__device__ __forceinline__ int num_kv_blocks1(const Params& p, int qb, bool causal) {
    return causal ? min(p.num_kblocks, qb + 1) : p.num_kblocks;
}

template <int D, bool kCausal>
__global__ void __launch_bounds__(kThreads, 1)
    fa_fwd_bf16_tile_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v, const Params p) {
    using L = Layout<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = ptx::smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    const uint32_t bar0 = base + L::kBarOff;
    auto q_full = [&](int b) { return bar0 + 8u * b; };
    auto q_empty = [&](int b) { return bar0 + 8u * (2 + b); };
    auto kv_full = [&](int s) { return bar0 + 8u * (4 + s); };
    auto kv_empty = [&](int s) { return bar0 + 8u * (4 + L::kSlots + s); };
    auto s_full = [&](int b) { return bar0 + 8u * (4 + 2 * L::kSlots + b); };
    // P of block g (the CTA's g-th block) is announced on p_full(g & 1): the
    // softmax warps may finish block g + 1 (its S was computed ahead) before
    // the MMA warp has seen block g, and one barrier would then complete two
    // phases unobserved.
    auto p_full = [&](uint32_t g) { return bar0 + 8u * (6 + 2 * L::kSlots + (g & 1u)); };
    const uint32_t pv_done = bar0 + 8u * (8 + 2 * L::kSlots);
    const uint32_t o_free = pv_done + 8;
    auto sched_full = [&](int i) { return bar0 + 8u * (10 + 2 * L::kSlots + i); };
    auto sched_empty = [&](int i) { return bar0 + 8u * (10 + 2 * L::kSlots + kSchedDepth + i); };
    const uint32_t drain = bar0 + 8u * (10 + 2 * L::kSlots + 2 * kSchedDepth);
    auto pair_bar = [&](int q) { return drain + 8u * (1 + q); };

    uint32_t* tmem_base_ptr = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
    volatile int* unit_ring = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 8);
    const Sync sync{abort_flag, p.status};

    if (threadIdx.x == 0) {
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(q_full(b), 1);
            ptx::mbar_init(q_empty(b), 1);
            ptx::mbar_init(s_full(b), 1);
        }
        for (int s = 0; s < L::kSlots; ++s) {
            ptx::mbar_init(kv_full(s), 1);
            ptx::mbar_init(kv_empty(s), 1);
        }
        ptx::mbar_init(p_full(0), 32 * kSoftmaxWarps);
        ptx::mbar_init(p_full(1), 32 * kSoftmaxWarps);
        ptx::mbar_init(pv_done, 1);
        ptx::mbar_init(o_free, 32 * kSoftmaxWarps);
        for (int i = 0; i < kSchedDepth; ++i) {
            ptx::mbar_init(sched_full(i), 1);
            ptx::mbar_init(sched_empty(i), 1 + kSoftmaxWarps);
        }
        ptx::mbar_init(drain, 1);
        for (int q = 0; q < 4; ++q) ptx::mbar_init(pair_bar(q), 64);
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
        // K/V tiles in the order the MMA warp consumes them: K_0, K_1, then
        // V_j followed by K_{j+2} for each block j.
        const bool leader = ptx::elect_one();
        const uint64_t keep = ptx::policy_evict_last();
        const uint64_t once = ptx::policy_evict_first();
        int slot = 0;
        uint32_t phase = 0, nloads = 0;
        uint32_t q_issued[2] = {0, 0};
        bool ok = true;
        auto load_kv = [&](const CUtensorMap* tm, int j, int bh) {
            ok = __all_sync(0xffffffffu, tc::wait_bar(sync, kv_empty(slot), phase ^ 1));
            if (!ok) return;
            const uint32_t dst = base + L::kRingOff + slot * L::kTileBytes;
            if (leader) {
                ptx::mbar_arrive_expect_tx(kv_full(slot), L::kTileBytes);
                for (int h = 0; h < L::kHalves; ++h)
                    ptx::tma_load_3d(dst + h * L::kPanelBytes, tm, kv_full(slot), h * 64, j * kBlockN, bh, keep);
            }
            ++nloads;
            if (++slot == L::kSlots) {
                slot = 0;
                phase ^= 1;
            }
        };
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
            const Unit w = tc::decode_unit(u, p, kCausal);
            const int n = num_kv_blocks1(p, w.qb, kCausal);
            const int qb_ = it & 1;
            ok = __all_sync(0xffffffffu, tc::wait_bar(sync, q_empty(qb_), ((it >> 1) & 1) ^ 1));
            if (!ok) break;
            const bool skip = p.skip_one_arrival && blockIdx.x == 0 && it == 0;
            if (!skip) {
                q_issued[qb_] = ((it >> 1) & 1) + 1;
                if (leader) {
                    ptx::mbar_arrive_expect_tx(q_full(qb_), L::kTileBytes);
                    for (int h = 0; h < L::kHalves; ++h)
                        ptx::tma_load_3d(base + L::kQOff + qb_ * L::kTileBytes + h * L::kPanelBytes, &tm_q, q_full(qb_),
                                         h * 64, w.qb * kBlockM, w.bh, once);
                }
            }
            load_kv(&tm_k, 0, w.bh);
            if (ok && n > 1) load_kv(&tm_k, 1, w.bh);
            for (int j = 0; j < n && ok; ++j) {
                load_kv(&tm_v, j, w.bh);
                if (ok && j + 2 < n) load_kv(&tm_k, j + 2, w.bh);
            }
        }
        for (uint32_t s = 0; s < static_cast<uint32_t>(L::kSlots) && s < nloads; ++s) {
            const uint32_t last = s + L::kSlots * ((nloads - 1 - s) / L::kSlots);
            tc::drain_bar(sync, kv_full(s), (last / L::kSlots) & 1);
        }
        for (int b = 0; b < 2; ++b)
            if (q_issued[b]) tc::drain_bar(sync, q_full(b), q_issued[b] - 1);
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
        // Per unit of n blocks: S_0, S_1, then for each block j: P_j V_j and
        // S_{j+2}.  S_j lives in TMEM buffer (c + j) & 1 (c counts the CTA's
        // earlier blocks); P_j is written over it, and S_{j+2} reuses the
        // buffer once P_j V_j has read it (one thread's MMAs run in order).
        const bool leader = ptx::elect_one();
        constexpr uint32_t idesc_s = ptx::make_idesc_bf16(kBlockM, kBlockN, false);
        constexpr uint32_t idesc_o = ptx::make_idesc_bf16(kBlockM, D, true);
        const uint64_t desc_q0 = ptx::make_smem_desc(base + L::kQOff, 16, 1024);
        const uint64_t desc_k0 = ptx::make_smem_desc(base + L::kRingOff, 16, 1024);
        const uint64_t desc_v0 = ptx::make_smem_desc(base + L::kRingOff, L::kPanelBytes, 1024);
        int slot = 0;
        uint32_t phase = 0;
        uint32_t sc = 0;   // S tiles issued by this CTA
        uint32_t pc = 0;   // blocks whose P has been consumed
        uint32_t units_done = 0;
        bool ok = true;
        auto commit = [&](uint32_t bar) {
            if (leader) ptx::mma_commit(bar);
        };
        auto wait_all = [&](uint32_t bar, uint32_t parity) {
            return __all_sync(0xffffffffu, tc::wait_bar(sync, bar, parity));
        };
        auto next_slot = [&](int& s, uint32_t& ph) {
            s = slot;
            ph = phase;
            if (++slot == L::kSlots) {
                slot = 0;
                phase ^= 1;
            }
        };
        auto issue_s = [&](int qbuf) {
            int sk;
            uint32_t pk;
            next_slot(sk, pk);
            ok = wait_all(kv_full(sk), pk);
            if (!ok) return;
            ptx::tc_fence_after_sync();
            const uint32_t sbuf = sc & 1u;
            const uint64_t qd = desc_q0 + ((qbuf * L::kTileBytes) >> 4);
            const uint64_t kd = desc_k0 + ((sk * L::kTileBytes) >> 4);
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const uint32_t off = ((ks >> 2) * L::kPanelBytes + (ks & 3) * 32) >> 4;
                if (leader) ptx::mma_ss(tmem + L::kTmemS + 128 * sbuf, qd + off, kd + off, idesc_s, ks > 0);
            }
            commit(s_full(sbuf));
            commit(kv_empty(sk));
            ++sc;
        };
        for (uint32_t it = 0; ok; ++it) {
            const int rs = it % kSchedDepth;
            ok = wait_all(sched_full(rs), (it / kSchedDepth) & 1);
            if (!ok) break;
            const int u = unit_ring[rs];
            __syncwarp();
            if (leader) ptx::mbar_arrive(sched_empty(rs));
            if (u < 0) break;
            const Unit w = tc::decode_unit(u, p, kCausal);
            const int n = num_kv_blocks1(p, w.qb, kCausal);
            const int qbuf = it & 1;
            ok = wait_all(q_full(qbuf), (it >> 1) & 1);
            if (!ok) break;
            const uint32_t c0 = sc;  // S number of block 0 of this unit
            issue_s(qbuf);
            if (ok && n > 1) issue_s(qbuf);
            if (ok && n <= 2) commit(q_empty(qbuf));
            for (int j = 0; j < n && ok; ++j) {
                int sv;
                uint32_t pvph;
                next_slot(sv, pvph);
                ok = wait_all(kv_full(sv), pvph);
                if (!ok) break;
                ok = wait_all(p_full(pc), (pc >> 1) & 1u);
                if (!ok) break;
                ++pc;
                if (j == 0 && units_done > 0) {
                    ok = wait_all(o_free, (units_done - 1) & 1u);  // the previous unit's O has been read
                    if (!ok) break;
                }
                ptx::tc_fence_after_sync();
                const uint32_t sbuf = (c0 + j) & 1u;
                const uint64_t vd = desc_v0 + ((sv * L::kTileBytes) >> 4);
#pragma unroll
                for (int ks = 0; ks < kBlockN / 16; ++ks) {
                    if (leader)
                        ptx::mma_ts(tmem + L::kTmemO, tmem + L::kTmemS + 128 * sbuf + ks * 8,
                                    vd + ((ks * 16 * 128) >> 4), idesc_o, (j > 0 || ks > 0) ? 1u : 0u);
                }
                commit(kv_empty(sv));
                commit(pv_done);
                if (j + 2 < n) {
                    issue_s(qbuf);
                    if (ok && j + 2 == n - 1) commit(q_empty(qbuf));
                }
            }
            ++units_done;
        }
        commit(drain);
        tc::drain_bar(sync, drain, 0);
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax warps
        // The two warps sharing TMEM lane quarter q split its 32 rows (half h:
        // rows 32q + 16h .. +15), read with the 16-lane shapes; a quad of
        // threads owns two rows, r0 and r0 + 8, and in every 8-column chunk k
        // the column pair 8k + 2(lane % 4) + {0, 1}.
        const int q = warp & 3;
        const int h = warp >> 2;
        const int qc = lane & 3;
        const int rr0 = 32 * q + 16 * h + (lane >> 2);
        const uint32_t lane_addr = static_cast<uint32_t>(32 * q + 16 * h) << 16;
        const uint32_t tmem_o = tmem + lane_addr + L::kTmemO;
        const uint32_t tmem_o_rows = tmem + (static_cast<uint32_t>(32 * q) << 16) + L::kTmemO;
        float* inv_l_base = reinterpret_cast<float*>(smem + L::kInvLOff);
        const float sl = p.scale_log2;
        uint32_t sc = 0;   // S tiles consumed (the MMA warp's numbering)
        uint32_t pair_phase = 0;
        int buf = 0;
        bool ok = true;

        for (uint32_t it = 0; ok; ++it) {
            const int rs = it % kSchedDepth;
            ok = __all_sync(0xffffffffu, tc::wait_bar(sync, sched_full(rs), (it / kSchedDepth) & 1));
            if (!ok) break;
            const int u = unit_ring[rs];
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(sched_empty(rs));
            if (u < 0) break;

            const Unit w = tc::decode_unit(u, p, kCausal);
            const int n = num_kv_blocks1(p, w.qb, kCausal);
            const int tile_row0 = w.qb * kBlockM;
            const int row0 = tile_row0 + rr0;
            const int row1 = row0 + 8;
            float m_run[2] = {-INFINITY, -INFINITY};
            float l_run[2] = {0.f, 0.f};
            float lb_run[2] = {0.f, 0.f};

            for (int j = 0; j < n; ++j) {
                const uint32_t sbuf = sc & 1u;
                ok = __all_sync(0xffffffffu, tc::wait_bar(sync, s_full(sbuf), (sc >> 1) & 1u));
                if (!ok) break;
                ++sc;
                ptx::tc_fence_after_sync();
                const uint32_t tmem_s = tmem + lane_addr + L::kTmemS + 128 * sbuf;

                const int key0 = j * kBlockN;
                const bool need_mask = (key0 + kBlockN > p.n) || (kCausal && key0 + kBlockN - 1 > tile_row0);
                const float slv = need_mask ? 1.f : sl;
                uint32_t sr[64];
                float(&s)[64] = *reinterpret_cast<float(*)[64]>(sr);
                auto load_scores = [&]() {
                    ptx::tmem_ld16x256b_x16_wait(tmem_s, sr);
                    if (need_mask) {
                        const int lim0 = kCausal ? min(p.n - 1, row0) : (p.n - 1);
                        const int lim1 = kCausal ? min(p.n - 1, row1) : (p.n - 1);
#pragma unroll
                        for (int k = 0; k < 16; ++k)
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const int key = key0 + 8 * k + 2 * qc + (i & 1);
                                const int lim = (i < 2) ? lim0 : lim1;
                                s[4 * k + i] = (key <= lim) ? s[4 * k + i] * sl : -INFINITY;
                            }
                    }
                };
                auto block_max = [&](float (&mx)[2]) {
                    if (slv >= 0.f)
                        tc::quad_row_extreme<true>(s, mx);
                    else
                        tc::quad_row_extreme<false>(s, mx);
                    mx[0] *= slv;
                    mx[1] *= slv;
                };
                uint32_t pk[32];
                float a[2][2], b[2][2];
                auto exponentiate = [&](const float (&neg_m)[2]) {
#pragma unroll
                    for (int r = 0; r < 2; ++r) a[r][0] = a[r][1] = b[r][0] = b[r][1] = 0.f;
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
#pragma unroll
                        for (int r = 0; r < 2; ++r) {
                            float x0, x1;
                            ptx::fma2(x0, x1, s[4 * k + 2 * r], s[4 * k + 2 * r + 1], slv, slv, neg_m[r], neg_m[r]);
                            const float p0 = ptx::ex2(x0), p1 = ptx::ex2(x1);
                            const uint32_t v = ptx::pack_bf16x2(p0, p1);
                            pk[2 * k + r] = v;
                            ptx::add2(a[r][0], a[r][1], a[r][0], a[r][1], p0, p1);
                            ptx::add_bf16x2_to_f32(b[r][0], b[r][1], v);
                        }
                    }
                };
                auto neg_of = [](float m) { return (m == -INFINITY) ? 0.f : -m; };

                load_scores();
                float alpha[2] = {1.f, 1.f};
                bool rescale_o = false;
                if (j == 0) {
                    float mx[2];
                    block_max(mx);
                    m_run[0] = mx[0];
                    m_run[1] = mx[1];
                    const float nm[2] = {neg_of(m_run[0]), neg_of(m_run[1])};
                    exponentiate(nm);
                } else {
                    const float nm[2] = {neg_of(m_run[0]), neg_of(m_run[1])};
                    exponentiate(nm);
                    const bool big = (a[0][0] + a[0][1] > kStaleMaxBound) || (a[1][0] + a[1][1] > kStaleMaxBound);
                    if (__any_sync(0xffffffffu, big)) {
                        load_scores();
                        float mx[2];
                        block_max(mx);
#pragma unroll
                        for (int r = 0; r < 2; ++r) {
                            if (mx[r] > m_run[r]) {
                                alpha[r] = ptx::ex2(m_run[r] - mx[r]);
                                m_run[r] = mx[r];
                                rescale_o = true;
                            }
                        }
                        const float nm2[2] = {neg_of(m_run[0]), neg_of(m_run[1])};
                        exponentiate(nm2);
                    }
                }
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    l_run[r] = l_run[r] * alpha[r] + (a[r][0] + a[r][1]);
                    lb_run[r] = lb_run[r] * alpha[r] + (b[r][0] + b[r][1]);
                }
                ptx::tmem_st16x128b_x16(tmem_s, pk);
                // P_{j-1} V is complete before O is touched or P_j released
                // (its S tile was issued earlier, so S_j's completion does not
                // imply it).  Each P V completion is observed exactly once.
                if (j > 0) {
                    ok = __all_sync(0xffffffffu, tc::wait_bar(sync, pv_done, (sc - 2) & 1u));
                    if (!ok) break;
                    ptx::tc_fence_after_sync();
                }
                if (__any_sync(0xffffffffu, rescale_o)) {
#pragma unroll
                    for (int c0 = 0; c0 < D; c0 += 32) {
                        uint32_t ov[16];
                        ptx::tmem_ld16x256b_x4_wait(tmem_o + c0, ov);
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha[(i >> 1) & 1]);
                        ptx::tmem_st16x256b_x4(tmem_o + c0, ov);
                    }
                }
                ptx::tmem_st_wait();
                ptx::tc_fence_before_sync();
                ptx::mbar_arrive(p_full(sc - 1));
            }
            if (!ok) break;

            // End of the unit: row sums across the quad, 1/l shared with the
            // other warp of the lane quarter, lse written once.
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 1);
                l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 2);
                lb_run[r] += __shfl_xor_sync(0xffffffffu, lb_run[r], 1);
                lb_run[r] += __shfl_xor_sync(0xffffffffu, lb_run[r], 2);
            }
            float* inv_l_sm = inv_l_base + buf * kBlockM;
            if (qc == 0) {
                inv_l_sm[rr0] = 1.f / lb_run[0];
                inv_l_sm[rr0 + 8] = 1.f / lb_run[1];
                const float mu0 = (m_run[0] == -INFINITY) ? 0.f : m_run[0];
                const float mu1 = (m_run[1] == -INFINITY) ? 0.f : m_run[1];
                if (row0 < p.n) p.lse[static_cast<int64_t>(w.bh) * p.n + row0] = (mu0 + log2f(l_run[0])) * 0.69314718055994531f;
                if (row1 < p.n) p.lse[static_cast<int64_t>(w.bh) * p.n + row1] = (mu1 + log2f(l_run[1])) * 0.69314718055994531f;
            }
            ptx::mbar_arrive(pair_bar(q));
            ok = __all_sync(0xffffffffu, tc::wait_bar(sync, pair_bar(q), pair_phase));
            if (!ok) break;
            pair_phase ^= 1;
            // the unit's last P V, then O = O_acc / l: read, release O to the
            // next unit's first P V, then store from registers
            ok = __all_sync(0xffffffffu, tc::wait_bar(sync, pv_done, (sc - 1) & 1u));
            if (!ok) break;
            ptx::tc_fence_after_sync();
            uint32_t acc[D / 2];
            if constexpr (D == 128)
                ptx::tmem_ld64_wait(tmem_o_rows + (D / 2) * h, acc);
            else
                ptx::tmem_ld32_wait(tmem_o_rows + (D / 2) * h, acc);
            ptx::tc_fence_before_sync();
            ptx::mbar_arrive(o_free);
            const int row = tile_row0 + 32 * q + lane;
            const float inv_l = inv_l_sm[32 * q + lane];
            const bool valid = row < p.n;
            __nv_bfloat16* orow_g = p.o + (static_cast<int64_t>(w.bh) * p.n + row) * D + (D / 2) * h;
#pragma unroll
            for (int c0 = 0; c0 < D / 2; c0 += 32) {
                uint32_t packed[16];
#pragma unroll
                for (int c = 0; c < 32; c += 2)
                    packed[c >> 1] = ptx::pack_bf16x2(__uint_as_float(acc[c0 + c]) * inv_l,
                                                      __uint_as_float(acc[c0 + c + 1]) * inv_l);
                if (valid) {
                    uint4* dst = reinterpret_cast<uint4*>(orow_g + c0);
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
                }
            }
            buf ^= 1;
        }
        ptx::tc_fence_before_sync();
    }

    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    if (warp == kMmaWarp) {
        __syncwarp();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
    tc::clock_end(p, smem + L::kClockOff);
}

}  // namespace tc1
}  // namespace fa
