// fa_fwd_tc.cuh -- bf16 attention forward on the sm_100a tensor cores.
//
// What it computes (per head):  O = softmax(scale * Q K^T [causal]) V  and
// lse = ln(sum exp(scale * q.k)), exactly the attention of the pages
// (Chapter 15 -- FlashAttention, "Standard vs Flash Attention"), computed the
// way the FlashAttention column of that panel and "How It Works" describe:
// Q, K, V move in tiles from HBM to on-chip memory, S_tile = Q_tile K_tile^T
// and P_tile = softmax(S_tile) never leave the chip, O += P_tile V_tile
// accumulates, and O is written once.  The softmax is the online one with a
// running max m, a running sum l and a rescale of the accumulator when the
// max grows (FlashAttention, Playable, EP 04; Chapter 15, "Key Takeaways:
// Online Softmax Enables It").
//
// B200 mapping (not the pages' A100/H100 sketch):
//   * one CTA per SM, persistent; work units (b*h, 256-row query block) are
//     taken from a global queue in an order that keeps the units of a few
//     heads together (their K/V stay in L2) and, under the causal mask, runs
//     each group's heaviest query blocks first (Chapter 15, "FlashAttention
//     Evolution": work partitioning, persistent kernels);
//   * warp 9 is the TMA producer: it takes the next unit from the queue,
//     publishes it to the CTA through a shared-memory ring, loads the unit's
//     two Q tiles once and streams K_j, V_j through a ring of 128-row
//     shared-memory slots, all 128-byte swizzled;
//   * warp 8 issues tcgen05.mma from one thread: S_t = Q_t K_j^T into tensor
//     memory (TMEM), then O_t += P_t V_j with P_t read from TMEM;
//   * warps 0-3 and 4-7 are the softmax warpgroups for the unit's two query
//     tiles (t = 0, 1), one query row per thread: they read S_t from TMEM,
//     update m and l, write P_t (bf16) back over S_t, rescale O_t in TMEM when
//     the max grows past a threshold, and at the end normalise O_t and store
//     O and lse.  While one warpgroup exponentiates, the tensor core works on
//     the other tile.  Part of the exponentials run as a cubic polynomial on
//     the FMA pipe, because at d = 128 the special-function unit alone would
//     take as long as the tensor core.
//   * Causal: KV blocks entirely above the diagonal are never loaded or
//     multiplied; only the diagonal block is masked.
//
// TMEM columns (512 allocated): S_0/P_0 at 0, S_1/P_1 at 128, O_0 at 256,
// O_1 at 256 + D.  P_t (bf16 pairs) occupies the first 64 columns of S_t.
//
// Every mbarrier wait is bounded.  On expiry the waiting thread records
// kDevTimeout in the device status word and raises a CTA-wide abort flag;
// every role then leaves its loop, in-flight copies and MMAs are drained
// (again with bounded waits) and TMEM is freed before the CTA exits.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "sm100_ptx.cuh"

namespace fa {

constexpr int kDevTimeout = 1;  // value written to the device status word

namespace tc {

constexpr int kBlockM = 128;            // query rows per tile (one TMEM lane each)
constexpr int kBlockN = 128;            // keys per KV block
constexpr int kTilesPerUnit = 2;        // query tiles per work unit
constexpr int kUnitRows = kBlockM * kTilesPerUnit;
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp = 9;
constexpr int kThreads = 320;
constexpr int kSoftmaxWarps = 8;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;   // log2 units: rescale when the max grows by > 2^8
constexpr long long kWaitCycles = 1ll << 32;  // ~2 s at 2 GHz
constexpr int kSchedDepth = 2;              // unit ring between the producer and the other roles
constexpr int kHeadGroup = 8;               // heads whose units are interleaved in the queue
constexpr int kPolyPairsPer8 = 2;           // of every 8 column pairs, this many use exp2_poly2

template <int D>
struct Layout {
    static_assert(D == 64 || D == 128, "head dim");
    static constexpr int kHalves = D / 64;                     // 64-column (128-byte) swizzle panels
    static constexpr int kPanelBytes = kBlockM * 128;          // one panel of a 128-row tile
    static constexpr int kTileBytes = kPanelBytes * kHalves;   // a whole 128 x D bf16 tile
    static constexpr int kSlots = (D == 128) ? 4 : 8;          // K/V ring slots
    static constexpr int kQOff = 0;
    static constexpr int kRingOff = kQOff + kTilesPerUnit * kTileBytes;
    static constexpr int kBarOff = kRingOff + kSlots * kTileBytes;
    // barriers: q_full[2], q_empty[2], kv_full[S], kv_empty[S], s_full[2], p_full[2], o_full[2],
    //           sched_full[kSchedDepth], sched_empty[kSchedDepth], drain
    static constexpr int kNumBars = 2 + 2 + kSlots + kSlots + 2 + 2 + 2 + 2 * kSchedDepth + 1;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;    // tmem base, abort flag, unit ring
    static constexpr int kBytes = kMiscOff + 8 + 4 * kSchedDepth;
    static constexpr int kSmemBytes = kBytes + 1024;           // slack for 1024-byte alignment
    static constexpr uint32_t kTmemS = 0;
    static constexpr uint32_t kTmemO = 256;
};

struct Params {
    __nv_bfloat16* o;
    float* lse;
    int* status;         // device status word (kDevTimeout after a wait expired)
    unsigned* sched;     // [0] next unit, [1] CTAs finished; both back to 0 when the launch ends
    int bh;              // B * H
    int n;               // sequence length
    int num_qblocks;     // ceil(N / 256)
    int num_kblocks;     // ceil(N / 128)
    int num_units;       // bh * num_qblocks
    float scale_log2;    // scale * log2(e)
};

struct Sync {
    volatile int* abort;
    int* status;
};

// Give up: record the timeout once and tell the rest of the CTA.
__device__ __forceinline__ void raise_abort(const Sync& s) {
    if (*s.abort == 0) {
        *s.abort = 1;
        atomicCAS(s.status, 0, kDevTimeout);
    }
}

// Bounded wait for phase `parity` of `bar`.  False when the CTA is aborting.
__device__ __forceinline__ bool wait_bar(const Sync& s, uint32_t bar, uint32_t parity) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if (*s.abort) return false;
        if (clock64() - t0 > kWaitCycles) {
            raise_abort(s);
            return false;
        }
    }
}

// Bounded wait used while draining: ignores the abort flag.
__device__ __forceinline__ void drain_bar(const Sync& s, uint32_t bar, uint32_t parity) {
    const long long t0 = clock64();
    while (!ptx::mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > kWaitCycles) {
            raise_abort(s);
            return;
        }
    }
}

// Queue position -> (bh, query block).  Heads go in groups of kHeadGroup;
// inside a group the units of its heads are interleaved by query block, and
// under the causal mask the last (heaviest) query blocks come first.
struct Unit {
    int bh, qb;
};
__device__ __forceinline__ Unit decode_unit(int u, const Params& p, bool causal) {
    const int per_group = kHeadGroup * p.num_qblocks;
    const int g = u / per_group;
    const int r = u - g * per_group;
    const int hg = min(kHeadGroup, p.bh - g * kHeadGroup);
    const int qi = r / hg;
    Unit w;
    w.bh = g * kHeadGroup + (r - qi * hg);
    w.qb = causal ? (p.num_qblocks - 1 - qi) : qi;
    return w;
}

// KV blocks tile t of query block qb must visit.
__device__ __forceinline__ int num_kv_blocks(const Params& p, int qb, int t, bool causal) {
    if (!causal) return p.num_kblocks;
    const int last = qb * (kUnitRows / kBlockN) + t;  // the diagonal block
    return min(p.num_kblocks, last + 1);
}

// One block of the online softmax for this thread's row: x_c = s_c * slv - m
// (log2 units), p_c = 2^x_c packed to bf16 pairs, and two row sums -- in fp32
// (for lse) and of the bf16-rounded p that enters P V (for normalising O, so
// that O = sum(p v) / sum(p) with the same p on both sides).
template <bool kPoly>
__device__ __forceinline__ void exp_block(const float (&s)[kBlockN], float slv, float m_use,
                                          uint32_t (&pk)[kBlockN / 2], float& sum, float& sum_bf16) {
    float a[4][2] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
    float b[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
    const float neg_m = -m_use;
#pragma unroll
    for (int pi = 0; pi < kBlockN / 2; ++pi) {
        float x0, x1, p0, p1;
        ptx::fma2(x0, x1, s[2 * pi], s[2 * pi + 1], slv, slv, neg_m, neg_m);
        if (kPoly && (pi & 7) < kPolyPairsPer8) {
            ptx::exp2_poly2(p0, p1, x0, x1);
        } else {
            p0 = ptx::ex2(x0);
            p1 = ptx::ex2(x1);
        }
        pk[pi] = ptx::pack_bf16x2(p0, p1);
        ptx::add2(a[pi & 3][0], a[pi & 3][1], a[pi & 3][0], a[pi & 3][1], p0, p1);
        ptx::add_bf16x2_to_f32(b[pi & 1][0], b[pi & 1][1], pk[pi]);
    }
    sum = ((a[0][0] + a[0][1]) + (a[1][0] + a[1][1])) + ((a[2][0] + a[2][1]) + (a[3][0] + a[3][1]));
    sum_bf16 = (b[0][0] + b[0][1]) + (b[1][0] + b[1][1]);
}

// Row max (or min) of 128 values: eight independent chains of three-input ops.
template <bool kMax>
__device__ __forceinline__ float reduce_row(const float (&s)[kBlockN]) {
    float r[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float acc = s[16 * i];
#pragma unroll
        for (int c = 1; c < 15; c += 2)
            acc = kMax ? ptx::max3(acc, s[16 * i + c], s[16 * i + c + 1])
                       : ptx::min3(acc, s[16 * i + c], s[16 * i + c + 1]);
        r[i] = kMax ? fmaxf(acc, s[16 * i + 15]) : fminf(acc, s[16 * i + 15]);
    }
    if (kMax) return fmaxf(ptx::max3(r[0], r[1], r[2]), ptx::max3(r[3], r[4], ptx::max3(r[5], r[6], r[7])));
    return fminf(ptx::min3(r[0], r[1], r[2]), ptx::min3(r[3], r[4], ptx::min3(r[5], r[6], r[7])));
}

template <int D, bool kCausal>
__global__ void __launch_bounds__(kThreads, 1)
    fa_fwd_bf16_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const Params p) {
    using L = Layout<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = ptx::smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // barrier addresses
    const uint32_t bar0 = base + L::kBarOff;
    auto q_full = [&](int t) { return bar0 + 8u * t; };
    auto q_empty = [&](int t) { return bar0 + 8u * (2 + t); };
    auto kv_full = [&](int s) { return bar0 + 8u * (4 + s); };
    auto kv_empty = [&](int s) { return bar0 + 8u * (4 + L::kSlots + s); };
    auto s_full = [&](int t) { return bar0 + 8u * (4 + 2 * L::kSlots + t); };
    auto p_full = [&](int t) { return bar0 + 8u * (6 + 2 * L::kSlots + t); };
    auto o_full = [&](int t) { return bar0 + 8u * (8 + 2 * L::kSlots + t); };
    auto sched_full = [&](int i) { return bar0 + 8u * (10 + 2 * L::kSlots + i); };
    auto sched_empty = [&](int i) { return bar0 + 8u * (10 + 2 * L::kSlots + kSchedDepth + i); };
    const uint32_t drain = bar0 + 8u * (10 + 2 * L::kSlots + 2 * kSchedDepth);

    uint32_t* tmem_base_ptr = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
    volatile int* unit_ring = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 8);
    const Sync sync{abort_flag, p.status};

    if (threadIdx.x == 0) {
        for (int t = 0; t < 2; ++t) {
            ptx::mbar_init(q_full(t), 1);
            ptx::mbar_init(q_empty(t), 1);
            ptx::mbar_init(s_full(t), 1);
            ptx::mbar_init(p_full(t), kBlockM);
            ptx::mbar_init(o_full(t), 1);
        }
        for (int s = 0; s < L::kSlots; ++s) {
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
    const uint32_t tmem = *tmem_base_ptr;

    if (warp == kLoadWarp) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t keep = ptx::policy_evict_last();   // K/V: re-read by the head's other units
            const uint64_t once = ptx::policy_evict_first();  // Q: read once
            int slot = 0;
            uint32_t phase = 0;
            // last issued phase per slot (+1), for draining
            uint32_t slot_issued[L::kSlots];
            uint32_t q_issued[2] = {0, 0};
            for (int s = 0; s < L::kSlots; ++s) slot_issued[s] = 0;
            bool ok = true;
            for (uint32_t it = 0; ok; ++it) {
                // take the next unit from the queue and publish it to the CTA
                const int rs = it % kSchedDepth;
                ok = wait_bar(sync, sched_empty(rs), ((it / kSchedDepth) & 1) ^ 1);
                if (!ok) break;
                int u = static_cast<int>(atomicAdd(p.sched, 1u));
                if (u >= p.num_units) u = -1;
                unit_ring[rs] = u;
                ptx::mbar_arrive(sched_full(rs));
                if (u < 0) break;

                const Unit w = decode_unit(u, p, kCausal);
                const int n1 = num_kv_blocks(p, w.qb, 1, kCausal);
                for (int t = 0; t < 2 && ok; ++t) {
                    ok = wait_bar(sync, q_empty(t), (it & 1) ^ 1);
                    if (!ok) break;
                    const uint32_t dst = base + L::kQOff + t * L::kTileBytes;
                    ptx::mbar_arrive_expect_tx(q_full(t), L::kTileBytes);
                    q_issued[t] = (it & 1) + 1;
                    for (int h = 0; h < L::kHalves; ++h)
                        ptx::tma_load_3d(dst + h * L::kPanelBytes, &tm_q, q_full(t), h * 64,
                                         w.qb * kUnitRows + t * kBlockM, w.bh, once);
                }
                for (int j = 0; j < n1 && ok; ++j) {
                    for (int kv = 0; kv < 2 && ok; ++kv) {
                        ok = wait_bar(sync, kv_empty(slot), phase ^ 1);
                        if (!ok) break;
                        const uint32_t dst = base + L::kRingOff + slot * L::kTileBytes;
                        ptx::mbar_arrive_expect_tx(kv_full(slot), L::kTileBytes);
                        slot_issued[slot] = phase + 1;
                        const CUtensorMap* tm = kv == 0 ? &tm_k : &tm_v;
                        for (int h = 0; h < L::kHalves; ++h)
                            ptx::tma_load_3d(dst + h * L::kPanelBytes, tm, kv_full(slot), h * 64,
                                             j * kBlockN, w.bh, keep);
                        if (++slot == L::kSlots) {
                            slot = 0;
                            phase ^= 1;
                        }
                    }
                }
            }
            // Drain: every issued copy must land before shared memory is released.
            for (int s = 0; s < L::kSlots; ++s)
                if (slot_issued[s]) drain_bar(sync, kv_full(s), slot_issued[s] - 1);
            for (int t = 0; t < 2; ++t)
                if (q_issued[t]) drain_bar(sync, q_full(t), q_issued[t] - 1);
            // The last CTA to finish returns the queue to zero for the next launch.
            __threadfence();
            if (atomicAdd(p.sched + 1, 1u) == gridDim.x - 1) {
                atomicExch(p.sched, 0u);
                atomicExch(p.sched + 1, 0u);
            }
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = ptx::make_idesc_bf16(kBlockM, kBlockN, false);
            constexpr uint32_t idesc_o = ptx::make_idesc_bf16(kBlockM, D, true);
            int slot = 0;
            uint32_t phase = 0;
            uint32_t p_phase[2] = {0, 0};
            bool ok = true;

            // S_t = Q_t K^T over the head dim: D/16 MMAs of K = 16.
            auto issue_s = [&](int t, int kslot) {
                const uint32_t q_base = base + L::kQOff + t * L::kTileBytes;
                const uint32_t k_base = base + L::kRingOff + kslot * L::kTileBytes;
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t off = (ks >> 2) * L::kPanelBytes + (ks & 3) * 32;
                    const uint64_t a = ptx::make_smem_desc(q_base + off, 16, 1024);
                    const uint64_t b = ptx::make_smem_desc(k_base + off, 16, 1024);
                    ptx::mma_ss(tmem + L::kTmemS + t * kBlockN, a, b, idesc_s, ks > 0);
                }
            };
            // O_t (+)= P_t V: 128/16 MMAs; P from TMEM (8 columns per 16 keys),
            // V from shared memory as an MN-major operand (d contiguous).
            auto issue_pv = [&](int t, int vslot, bool accumulate) {
                const uint32_t v_base = base + L::kRingOff + vslot * L::kTileBytes;
#pragma unroll
                for (int ks = 0; ks < kBlockN / 16; ++ks) {
                    const uint64_t b = ptx::make_smem_desc(v_base + ks * 16 * 128, L::kPanelBytes, 1024);
                    ptx::mma_ts(tmem + L::kTmemO + t * D, tmem + L::kTmemS + t * kBlockN + ks * 8, b,
                                idesc_o, (accumulate || ks > 0) ? 1u : 0u);
                }
            };
            auto next_slot = [&](int& s, uint32_t& ph) {
                s = slot;
                ph = phase;
                if (++slot == L::kSlots) {
                    slot = 0;
                    phase ^= 1;
                }
            };

            for (uint32_t it = 0; ok; ++it) {
                const int rs = it % kSchedDepth;
                ok = wait_bar(sync, sched_full(rs), (it / kSchedDepth) & 1);
                if (!ok) break;
                const int u = unit_ring[rs];
                ptx::mbar_arrive(sched_empty(rs));
                if (u < 0) break;

                const Unit w = decode_unit(u, p, kCausal);
                const int n0 = num_kv_blocks(p, w.qb, 0, kCausal);
                const int n1 = num_kv_blocks(p, w.qb, 1, kCausal);
                ok = wait_bar(sync, q_full(0), it & 1) && wait_bar(sync, q_full(1), it & 1);
                if (!ok) break;
                int sk, sv;
                uint32_t pk, pv;
                next_slot(sk, pk);
                ok = wait_bar(sync, kv_full(sk), pk);
                if (!ok) break;
                ptx::tc_fence_after_sync();
                issue_s(0, sk);
                ptx::mma_commit(s_full(0));
                if (n0 == 1) ptx::mma_commit(q_empty(0));
                issue_s(1, sk);
                ptx::mma_commit(s_full(1));
                if (n1 == 1) ptx::mma_commit(q_empty(1));
                ptx::mma_commit(kv_empty(sk));

                for (int j = 0; j < n1 && ok; ++j) {
                    next_slot(sv, pv);
                    ok = wait_bar(sync, kv_full(sv), pv);
                    if (!ok) break;
                    if (j < n0) {
                        ok = wait_bar(sync, p_full(0), p_phase[0]);
                        if (!ok) break;
                        p_phase[0] ^= 1;
                        ptx::tc_fence_after_sync();
                        issue_pv(0, sv, j > 0);
                        if (j == n0 - 1) ptx::mma_commit(o_full(0));
                    }
                    const bool more = j + 1 < n1;
                    if (more) {
                        next_slot(sk, pk);
                        ok = wait_bar(sync, kv_full(sk), pk);
                        if (!ok) break;
                        ptx::tc_fence_after_sync();
                    }
                    if (j + 1 < n0) {
                        issue_s(0, sk);
                        ptx::mma_commit(s_full(0));
                        if (j + 1 == n0 - 1) ptx::mma_commit(q_empty(0));
                    }
                    ok = wait_bar(sync, p_full(1), p_phase[1]);
                    if (!ok) break;
                    p_phase[1] ^= 1;
                    ptx::tc_fence_after_sync();
                    issue_pv(1, sv, j > 0);
                    if (j == n1 - 1) ptx::mma_commit(o_full(1));
                    ptx::mma_commit(kv_empty(sv));
                    if (more) {
                        issue_s(1, sk);
                        ptx::mma_commit(s_full(1));
                        if (j + 1 == n1 - 1) ptx::mma_commit(q_empty(1));
                        ptx::mma_commit(kv_empty(sk));
                    }
                }
            }
            // Drain: all issued MMAs complete before TMEM is released.
            ptx::mma_commit(drain);
            drain_bar(sync, drain, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax warpgroups
        const int t = warp >> 2;                         // query tile of this warpgroup
        const int row_in_tile = (warp & 3) * 32 + lane;  // TMEM lane == tile row
        const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tmem_s = tmem + lane_addr + L::kTmemS + t * kBlockN;
        const uint32_t tmem_o = tmem + lane_addr + L::kTmemO + t * D;
        const float sl = p.scale_log2;
        uint32_t s_phase = 0, o_phase = 0;
        bool ok = true;

        for (uint32_t it = 0; ok; ++it) {
            const int rs = it % kSchedDepth;
            ok = __all_sync(0xffffffffu, wait_bar(sync, sched_full(rs), (it / kSchedDepth) & 1));
            if (!ok) break;
            const int u = unit_ring[rs];
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(sched_empty(rs));
            if (u < 0) break;

            const Unit w = decode_unit(u, p, kCausal);
            const int nt = num_kv_blocks(p, w.qb, t, kCausal);
            const int tile_row0 = w.qb * kUnitRows + t * kBlockM;
            const int row = tile_row0 + row_in_tile;
            float m_run = -INFINITY;  // running max, log2 units (scale folded in)
            float l_run = 0.f;        // running sum of 2^(x - m_run), fp32
            float lb_run = 0.f;       // the same sum over the bf16-rounded values

            for (int j = 0; j < nt; ++j) {
                ok = __all_sync(0xffffffffu, wait_bar(sync, s_full(t), s_phase));
                if (!ok) break;
                s_phase ^= 1;
                ptx::tc_fence_after_sync();

                uint32_t sr[kBlockN];
                ptx::tmem_ld128_wait(tmem_s, sr);
                float(&s)[kBlockN] = *reinterpret_cast<float(*)[kBlockN]>(sr);

                const int key0 = j * kBlockN;
                const bool need_mask = (key0 + kBlockN > p.n) || (kCausal && key0 + kBlockN - 1 > tile_row0);
                float slv = sl;
                if (need_mask) {
                    // Masked block (diagonal or ragged tail): scores to log2 units
                    // and masked keys to -inf, whatever the sign of the scale.
                    const int limit = kCausal ? min(p.n - 1, row) : (p.n - 1);
#pragma unroll
                    for (int c = 0; c < kBlockN; ++c) s[c] = (key0 + c <= limit) ? s[c] * sl : -INFINITY;
                    slv = 1.f;
                }
                const float mx = slv >= 0.f ? reduce_row<true>(s) * slv : reduce_row<false>(s) * slv;

                // Online softmax update: raise the running max only when it
                // grows by more than the threshold (the result is exact either
                // way: O and l always share the same m).
                float alpha = 1.f;
                bool rescale_o = false;
                if (j == 0) {
                    m_run = mx;
                } else if (mx > m_run + kRescaleThreshold) {
                    alpha = ptx::ex2(m_run - mx);
                    m_run = mx;
                    rescale_o = true;
                }
                const float m_use = (m_run == -INFINITY) ? 0.f : m_run;

                uint32_t pk[kBlockN / 2];
                float rowsum, rowsum_bf16;
                if (need_mask)
                    exp_block<false>(s, slv, m_use, pk, rowsum, rowsum_bf16);
                else
                    exp_block<true>(s, slv, m_use, pk, rowsum, rowsum_bf16);
                l_run = l_run * alpha + rowsum;
                lb_run = lb_run * alpha + rowsum_bf16;
                ptx::tmem_st64(tmem_s, pk);

                // Rescale this row of O_t.  S_t(j) being complete means every
                // earlier MMA (PV_t(j-1) included) is complete, so O_t is stable.
                if (__any_sync(0xffffffffu, rescale_o)) {
#pragma unroll
                    for (int c0 = 0; c0 < D; c0 += 32) {
                        uint32_t orow[32];
                        ptx::tmem_ld32_wait(tmem_o + c0, orow);
#pragma unroll
                        for (int c = 0; c < 32; ++c)
                            orow[c] = __float_as_uint(__uint_as_float(orow[c]) * alpha);
                        ptx::tmem_st32(tmem_o + c0, orow);
                    }
                }
                ptx::tmem_st_wait();
                ptx::tc_fence_before_sync();
                ptx::mbar_arrive(p_full(t));
            }
            if (!ok) break;

            // Epilogue: O = O_acc / l, written once; lse in natural log.
            ok = __all_sync(0xffffffffu, wait_bar(sync, o_full(t), o_phase));
            if (!ok) break;
            o_phase ^= 1;
            ptx::tc_fence_after_sync();
            const float inv_l = 1.f / lb_run;
            const bool valid = row < p.n;
            __nv_bfloat16* orow_g = p.o + (static_cast<int64_t>(w.bh) * p.n + row) * D;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t acc[32];
                ptx::tmem_ld32_wait(tmem_o + c0, acc);
                uint32_t packed[16];
#pragma unroll
                for (int c = 0; c < 32; c += 2)
                    packed[c >> 1] = ptx::pack_bf16x2(__uint_as_float(acc[c]) * inv_l,
                                                      __uint_as_float(acc[c + 1]) * inv_l);
                if (valid) {
                    uint4* dst = reinterpret_cast<uint4*>(orow_g + c0);
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2],
                                            packed[4 * v + 3]);
                }
            }
            if (valid) {
                const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
                p.lse[static_cast<int64_t>(w.bh) * p.n + row] = (m_use + log2f(l_run)) * 0.69314718055994531f;
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
}

}  // namespace tc
}  // namespace fa
