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
//   * warp 17 is the TMA producer: it takes the next unit from the queue,
//     publishes it to the CTA through a shared-memory ring, loads the unit's
//     two Q tiles once and streams K_j, V_j through a ring of 128-row
//     shared-memory slots, all 128-byte swizzled;
//   * warp 16 issues tcgen05.mma from one elected lane: S_t = Q_t K_j^T into
//     tensor memory (TMEM), then O_t += P_t V_j with P_t read from TMEM;
//   * warps 0-7 and 8-15 are the softmax warps of the unit's two query tiles
//     (t = 0, 1), two warps per TMEM lane quarter, so a quad of threads owns
//     two rows: they read S_t from TMEM, update m and l, write P_t (bf16)
//     back over S_t, rescale O_t in TMEM when a block outgrows the running
//     max, and at the end of a unit write lse, normalise O_t by l and lay it
//     out in a shared-memory staging tile.  While one tile's warps
//     exponentiate, the tensor core works on the other tile.  At d = 128 the
//     exponentials on the special-function unit take about as long as the
//     tile's MMAs, so they are the co-limit of the kernel;
//   * warp 18 stores each staged O tile with a TMA tensor store (rows past
//     N are not written) and frees the staging tile once the store has read
//     it, so no softmax thread issues the 128 row-strided stores of a tile.
//   * Causal: KV blocks entirely above the diagonal are never loaded or
//     multiplied; only the diagonal block is masked.
//   * Launched with programmatic stream serialization: a CTA sets up its
//     barriers and TMEM while the previous kernel of the stream finishes and
//     waits for it (griddepcontrol.wait) before touching global memory.
//
// Small and medium problems can run the one-tile kernel of fa_fwd_tc1.cuh
// instead (same arithmetic, same results; the host picks by schedule).
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
constexpr int kSoftmaxWarps = 16;       // 8 per query tile
constexpr int kMmaWarp = 16;
constexpr int kLoadWarp = 17;
constexpr int kEpiWarp = 18;            // stores each finished tile of O with TMA
constexpr int kThreads = 608;
constexpr uint32_t kTmemCols = 512;
constexpr float kStaleMaxBound = 1048576.0f;  // 2^20: largest p accepted against a stale running max
constexpr long long kWaitCycles = 1ll << 32;  // ~2 s at 2 GHz
constexpr int kSchedDepth = 2;              // unit ring between the producer and the other roles
constexpr int kHeadGroup = 8;               // heads whose units are interleaved in the queue

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
    //           sched_full[kSchedDepth], sched_empty[kSchedDepth], drain, pair[2][4],
    //           stage_full[2], stage_free
    static constexpr int kNumBars = 2 + 2 + kSlots + kSlots + 2 + 2 + 2 + 2 * kSchedDepth + 1 + 8 + 3;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;    // tmem base, abort flag, unit ring, tile coordinates
    static constexpr int kInvLOff = (kMiscOff + 8 + 4 * kSchedDepth + 16 + 15) & ~15;  // float[2][128]
    static constexpr int kClockOff = kInvLOff + 2 * kBlockM * 4;                      // int64[2]: start clock, timer
    static constexpr int kStageOff = (kClockOff + 16 + 1023) & ~1023;   // one 128 x D bf16 O tile
    static constexpr int kBytes = kStageOff + kTileBytes;
    static constexpr int kSmemBytes = kBytes + 1024;           // slack for 1024-byte alignment
    static constexpr uint32_t kTmemS = 0;
    static constexpr uint32_t kTmemO = 256;
    static_assert(kSmemBytes <= 232448, "shared memory");
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
    int skip_one_arrival;  // test hook: CTA 0 never loads its first Q tile (one wait runs out)
    unsigned long long* clock;  // null, or [0] SM cycles, [1] timer ns, [2] CTAs: summed over CTAs
};

// Global timer in nanoseconds (%globaltimer).
__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Programmatic dependent launch (the kernels are launched with programmatic
// stream serialization): a CTA may start while the previous kernel of the
// stream is still running.  It sets up shared memory, barriers and tensor
// memory, then waits for that kernel to complete (and its writes to be
// visible) before it touches global memory; once its producer finds the work
// queue empty it lets the next kernel's CTAs start on SMs that free up.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void launch_dependents() { asm volatile("griddepcontrol.launch_dependents;"); }

// Clock record: each CTA adds the SM cycles and global-timer nanoseconds it
// ran, and one to the CTA count (the start values wait in shared memory).
__device__ __forceinline__ void clock_start(const Params& p, uint8_t* slot, bool me) {
    if (me && p.clock) {
        reinterpret_cast<long long*>(slot)[0] = clock64();
        reinterpret_cast<unsigned long long*>(slot)[1] = globaltimer();
    }
}
__device__ __forceinline__ void clock_end(const Params& p, const uint8_t* slot) {
    if (threadIdx.x == 0 && p.clock) {
        const long long c = clock64() - reinterpret_cast<const long long*>(slot)[0];
        const unsigned long long t = globaltimer() - reinterpret_cast<const unsigned long long*>(slot)[1];
        atomicAdd(p.clock, static_cast<unsigned long long>(c));
        atomicAdd(p.clock + 1, t);
        atomicAdd(p.clock + 2, 1ull);
    }
}

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

// Max (or min) of each of this thread's two rows (64 values in the .16x256b
// register order: 4k + {0,1} first row, 4k + {2,3} second row) completed
// across the quad that shares the rows.
template <bool kMax>
__device__ __forceinline__ void quad_row_extreme(const float (&s)[64], float (&out)[2]) {
    auto op = [](float a, float b) { return kMax ? fmaxf(a, b) : fminf(a, b); };
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        float c0 = s[2 * r], c1 = s[2 * r + 1], c2 = s[4 + 2 * r], c3 = s[5 + 2 * r];
#pragma unroll
        for (int k = 2; k < 16; k += 2) {
            c0 = op(c0, s[4 * k + 2 * r]);
            c1 = op(c1, s[4 * k + 2 * r + 1]);
            c2 = op(c2, s[4 * k + 4 + 2 * r]);
            c3 = op(c3, s[4 * k + 5 + 2 * r]);
        }
        out[r] = op(op(c0, c1), op(c2, c3));
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        out[r] = op(out[r], __shfl_xor_sync(0xffffffffu, out[r], 1));
        out[r] = op(out[r], __shfl_xor_sync(0xffffffffu, out[r], 2));
    }
}

template <int D, bool kCausal>
__global__ void __launch_bounds__(kThreads, 1)
    fa_fwd_bf16_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_o, const Params p) {
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
    // the two softmax warps of tile t that share TMEM lane quarter q meet here in the epilogue
    auto pair_bar = [&](int t, int q) { return bar0 + 8u * (11 + 2 * L::kSlots + 2 * kSchedDepth + 4 * t + q); };
    // the O staging tile: filled by tile t's softmax warps (stage_full(t)),
    // stored by the epilogue warp, free again once the store has read it
    auto stage_full = [&](int t) { return bar0 + 8u * (19 + 2 * L::kSlots + 2 * kSchedDepth + t); };
    const uint32_t stage_free = bar0 + 8u * (21 + 2 * L::kSlots + 2 * kSchedDepth);
    volatile int* stage_coord = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 8 + 4 * kSchedDepth);  // [t][bh, row0]

    uint32_t* tmem_base_ptr = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
    volatile int* unit_ring = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 8);
    const Sync sync{abort_flag, p.status};

    if (threadIdx.x == 0) {
        for (int t = 0; t < 2; ++t) {
            ptx::mbar_init(q_full(t), 1);
            ptx::mbar_init(q_empty(t), 1);
            ptx::mbar_init(s_full(t), 1);
            ptx::mbar_init(p_full(t), kSoftmaxWarps / 2);  // one arrival per warp
            for (int q = 0; q < 4; ++q) ptx::mbar_init(pair_bar(t, q), 64);
            ptx::mbar_init(o_full(t), 1);
        }
        for (int s = 0; s < L::kSlots; ++s) {
            ptx::mbar_init(kv_full(s), 1);
            ptx::mbar_init(kv_empty(s), 1);
        }
        for (int i = 0; i < kSchedDepth; ++i) {
            ptx::mbar_init(sched_full(i), 1);
            ptx::mbar_init(sched_empty(i), 2 + kSoftmaxWarps);
        }
        ptx::mbar_init(stage_full(0), 32 * (kSoftmaxWarps / 2));
        ptx::mbar_init(stage_full(1), 32 * (kSoftmaxWarps / 2));
        ptx::mbar_init(stage_free, 1);
        ptx::mbar_init(drain, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        ptx::tmem_alloc(ptx::smem_addr(tmem_base_ptr), kTmemCols);
        ptx::tmem_relinquish();
    }
    if (warp == kEpiWarp && lane == 0) ptx::prefetch_tmap(&tm_o);
    if (warp == kLoadWarp && lane == 0) {
        ptx::prefetch_tmap(&tm_q);
        ptx::prefetch_tmap(&tm_k);
        ptx::prefetch_tmap(&tm_v);
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    grid_dependency_wait();
    const uint32_t tmem = *tmem_base_ptr;

    if (warp == kLoadWarp) {
        clock_start(p, smem + L::kClockOff, lane == 0);
        // ------------------------------------------------------------ producer
        // The whole warp runs the loop (warp-uniform addresses and waits);
        // one elected lane issues the copies.
        const bool leader = ptx::elect_one();
        const uint64_t keep = ptx::policy_evict_last();   // K/V: re-read by the head's other units
        const uint64_t once = ptx::policy_evict_first();  // Q: read once
        int slot = 0;
        uint32_t phase = 0, nloads = 0;
        uint32_t q_issued[2] = {0, 0};  // last issued phase of each Q slot (+1), for draining
        bool ok = true;
        for (uint32_t it = 0; ok; ++it) {
            // take the next unit from the queue and publish it to the CTA
            const int rs = it % kSchedDepth;
            ok = __all_sync(0xffffffffu, wait_bar(sync, sched_empty(rs), ((it / kSchedDepth) & 1) ^ 1));
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
                launch_dependents();
                break;
            }

            const Unit w = decode_unit(u, p, kCausal);
            const int n1 = num_kv_blocks(p, w.qb, 1, kCausal);
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                if (!ok) break;
                ok = __all_sync(0xffffffffu, wait_bar(sync, q_empty(t), (it & 1) ^ 1));
                if (!ok) break;
                const uint32_t dst = base + L::kQOff + t * L::kTileBytes;
                if (p.skip_one_arrival && blockIdx.x == 0 && it == 0 && t == 0) continue;
                q_issued[t] = (it & 1) + 1;
                if (leader) {
                    ptx::mbar_arrive_expect_tx(q_full(t), L::kTileBytes);
                    for (int h = 0; h < L::kHalves; ++h)
                        ptx::tma_load_3d(dst + h * L::kPanelBytes, &tm_q, q_full(t), h * 64,
                                         w.qb * kUnitRows + t * kBlockM, w.bh, once);
                }
            }
            for (int j = 0; j < n1 && ok; ++j) {
                for (int kv = 0; kv < 2 && ok; ++kv) {
                    ok = __all_sync(0xffffffffu, wait_bar(sync, kv_empty(slot), phase ^ 1));
                    if (!ok) break;
                    const uint32_t dst = base + L::kRingOff + slot * L::kTileBytes;
                    if (leader) {
                        ptx::mbar_arrive_expect_tx(kv_full(slot), L::kTileBytes);
                        const CUtensorMap* tm = kv == 0 ? &tm_k : &tm_v;
                        for (int h = 0; h < L::kHalves; ++h)
                            ptx::tma_load_3d(dst + h * L::kPanelBytes, tm, kv_full(slot), h * 64,
                                             j * kBlockN, w.bh, keep);
                    }
                    ++nloads;
                    if (++slot == L::kSlots) {
                        slot = 0;
                        phase ^= 1;
                    }
                }
            }
        }
        // Drain: every issued copy must land before shared memory is released.
        // Load i went to slot i % S with phase (i / S) & 1.
        for (uint32_t s = 0; s < static_cast<uint32_t>(L::kSlots) && s < nloads; ++s) {
            const uint32_t last = s + L::kSlots * ((nloads - 1 - s) / L::kSlots);
            drain_bar(sync, kv_full(s), (last / L::kSlots) & 1);
        }
        for (int t = 0; t < 2; ++t)
            if (q_issued[t]) drain_bar(sync, q_full(t), q_issued[t] - 1);
        // The last CTA to finish returns the queue to zero for the next launch.
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
        // The whole warp runs the loop and builds the descriptors (so they are
        // warp-uniform); one elected lane issues every MMA and commit.
        const bool leader = ptx::elect_one();
        constexpr uint32_t idesc_s = ptx::make_idesc_bf16(kBlockM, kBlockN, false);
        constexpr uint32_t idesc_o = ptx::make_idesc_bf16(kBlockM, D, true);
        // base descriptors; operand offsets are added to the start-address field
        const uint64_t desc_q0 = ptx::make_smem_desc(base + L::kQOff, 16, 1024);
        const uint64_t desc_k0 = ptx::make_smem_desc(base + L::kRingOff, 16, 1024);
        const uint64_t desc_v0 = ptx::make_smem_desc(base + L::kRingOff, L::kPanelBytes, 1024);
        int slot = 0;
        uint32_t phase = 0;
        uint32_t p_phase[2] = {0, 0};
        bool ok = true;

        // S_t = Q_t K^T over the head dim: D/16 MMAs of K = 16.
        auto issue_s = [&](int t, int kslot) {
            const uint64_t qd = desc_q0 + ((t * L::kTileBytes) >> 4);
            const uint64_t kd = desc_k0 + ((kslot * L::kTileBytes) >> 4);
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const uint32_t off = ((ks >> 2) * L::kPanelBytes + (ks & 3) * 32) >> 4;
                if (leader) ptx::mma_ss(tmem + L::kTmemS + t * kBlockN, qd + off, kd + off, idesc_s, ks > 0);
            }
        };
        // O_t (+)= P_t V: 128/16 MMAs; P from TMEM (8 columns per 16 keys),
        // V from shared memory as an MN-major operand (d contiguous).
        auto issue_pv = [&](int t, int vslot, bool accumulate) {
            const uint64_t vd = desc_v0 + ((vslot * L::kTileBytes) >> 4);
#pragma unroll
            for (int ks = 0; ks < kBlockN / 16; ++ks) {
                if (leader)
                    ptx::mma_ts(tmem + L::kTmemO + t * D, tmem + L::kTmemS + t * kBlockN + ks * 8,
                                vd + ((ks * 16 * 128) >> 4), idesc_o, (accumulate || ks > 0) ? 1u : 0u);
            }
        };
        auto commit = [&](uint32_t bar) {
            if (leader) ptx::mma_commit(bar);
        };
        auto next_slot = [&](int& s, uint32_t& ph) {
            s = slot;
            ph = phase;
            if (++slot == L::kSlots) {
                slot = 0;
                phase ^= 1;
            }
        };
        auto wait_all = [&](uint32_t bar, uint32_t parity) {
            return __all_sync(0xffffffffu, wait_bar(sync, bar, parity));
        };

        // Unit `it` from the scheduling ring (-1: the queue is empty).
        auto fetch_unit = [&](uint32_t it, int& u) {
            const int rs = it % kSchedDepth;
            if (!wait_all(sched_full(rs), (it / kSchedDepth) & 1)) return false;
            u = unit_ring[rs];
            __syncwarp();
            if (leader) ptx::mbar_arrive(sched_empty(rs));
            return true;
        };
        // S_0(0) of a unit: Q_0 of that unit and its first K block.
        int sk = 0, sv = 0;
        uint32_t pk = 0, pv = 0;
        auto first_s0 = [&](uint32_t it, int n0) {
            if (!wait_all(q_full(0), it & 1)) return false;
            next_slot(sk, pk);
            if (!wait_all(kv_full(sk), pk)) return false;
            ptx::tc_fence_after_sync();
            issue_s(0, sk);
            commit(s_full(0));
            if (n0 == 1) commit(q_empty(0));
            return true;
        };

        int u = -1;
        ok = fetch_unit(0, u);
        bool s0_issued = false;  // S_0(0) of unit `it` went out during the previous unit
        for (uint32_t it = 0; ok && u >= 0; ++it) {
            const Unit w = decode_unit(u, p, kCausal);
            const int n0 = num_kv_blocks(p, w.qb, 0, kCausal);
            const int n1 = num_kv_blocks(p, w.qb, 1, kCausal);
            if (!s0_issued) {
                ok = first_s0(it, n0);
                if (!ok) break;
            }
            s0_issued = false;
            ok = wait_all(q_full(1), it & 1);
            if (!ok) break;
            ptx::tc_fence_after_sync();
            issue_s(1, sk);
            commit(s_full(1));
            if (n1 == 1) commit(q_empty(1));
            commit(kv_empty(sk));

            int next_u = -1;
            bool fetched = false;
            for (int j = 0; j < n1 && ok; ++j) {
                // V_j and K_{j+1} are waited for before P_0(j), so that PV_0(j)
                // and S_0(j+1) go to the tensor core back to back.
                next_slot(sv, pv);
                ok = wait_all(kv_full(sv), pv);
                if (!ok) break;
                const bool more = j + 1 < n1;
                if (more) {
                    next_slot(sk, pk);
                    ok = wait_all(kv_full(sk), pk);
                    if (!ok) break;
                }
                if (j < n0) {
                    ok = wait_all(p_full(0), p_phase[0]);
                    if (!ok) break;
                    p_phase[0] ^= 1;
                    ptx::tc_fence_after_sync();
                    issue_pv(0, sv, j > 0);
                    if (j == n0 - 1) commit(o_full(0));
                }
                if (j + 1 < n0) {
                    issue_s(0, sk);
                    commit(s_full(0));
                    if (j + 1 == n0 - 1) commit(q_empty(0));
                }
                if (!more) {
                    // Tile 0 is done with this unit: start the next unit's
                    // tile 0 now, so its warps find S_0(0) ready after their
                    // epilogue instead of waiting for tile 1's last block.
                    // (The ring holds this unit's last V, then the next
                    // unit's first K.)
                    ok = fetch_unit(it + 1, next_u);
                    if (!ok) break;
                    fetched = true;
                    if (next_u >= 0) {
                        const Unit wn = decode_unit(next_u, p, kCausal);
                        ok = first_s0(it + 1, num_kv_blocks(p, wn.qb, 0, kCausal));
                        if (!ok) break;
                        s0_issued = true;
                    }
                }
                ok = wait_all(p_full(1), p_phase[1]);
                if (!ok) break;
                p_phase[1] ^= 1;
                ptx::tc_fence_after_sync();
                issue_pv(1, sv, j > 0);
                if (j == n1 - 1) commit(o_full(1));
                commit(kv_empty(sv));
                if (more) {
                    issue_s(1, sk);
                    commit(s_full(1));
                    if (j + 1 == n1 - 1) commit(q_empty(1));
                    commit(kv_empty(sk));
                }
            }
            if (!ok) break;
            if (!fetched) {
                ok = fetch_unit(it + 1, next_u);
                if (!ok) break;
            }
            u = next_u;
        }
        // Drain: all issued MMAs complete before TMEM is released.
        commit(drain);
        drain_bar(sync, drain, 0);
        __syncwarp();
    } else if (warp == kEpiWarp) {
        // ------------------------------------------------------------ epilogue
        // For each unit, tile 0's then tile 1's O arrive in the staging tile;
        // one lane stores it with TMA (rows past N are not written) and, once
        // the store has read shared memory, frees the tile for the next one.
        bool ok = true;
        uint32_t uses = 0;
        for (uint32_t it = 0; ok; ++it) {
            const int rs = it % kSchedDepth;
            ok = __all_sync(0xffffffffu, wait_bar(sync, sched_full(rs), (it / kSchedDepth) & 1));
            if (!ok) break;
            const int u = unit_ring[rs];
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(sched_empty(rs));
            if (u < 0) break;
            for (int t = 0; t < 2 && ok; ++t, ++uses) {
                ok = __all_sync(0xffffffffu, wait_bar(sync, stage_full(t), it & 1));
                if (!ok) break;
                if (lane == 0) {
                    const int bh = stage_coord[2 * t], row0 = stage_coord[2 * t + 1];
                    for (int hh = 0; hh < L::kHalves; ++hh)
                        ptx::tma_store_3d(&tm_o, base + L::kStageOff + hh * L::kPanelBytes, hh * 64, row0, bh);
                    ptx::bulk_commit_group();
                    ptx::bulk_wait_group_read0();
                    ptx::mbar_arrive(stage_free);
                }
                __syncwarp();
            }
        }
        if (lane == 0) ptx::bulk_wait_group0();  // every store has landed
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax warps
        // Warps 0-7 serve query tile 0 and warps 8-15 tile 1.  The two warps
        // of a tile that share TMEM lane quarter q (= warp % 4) split its 32
        // rows: half h covers rows 32q + 16h .. +15, read with the 16-lane
        // TMEM shapes.  A quad of threads (lane / 4) owns two rows, r0 and
        // r0 + 8, and in every 8-column chunk k the column pair
        // 8k + 2(lane % 4) + {0, 1}; row reductions finish with two shuffles
        // inside the quad.
        const int t = warp >> 3;
        const int q = warp & 3;
        const int h = (warp >> 2) & 1;
        const int qc = lane & 3;                          // column pair within each chunk
        const int rr0 = 32 * q + 16 * h + (lane >> 2);    // row-in-tile of r0 (r1 = rr0 + 8)
        const uint32_t lane_addr = static_cast<uint32_t>(32 * q + 16 * h) << 16;
        const uint32_t tmem_s = tmem + lane_addr + L::kTmemS + t * kBlockN;
        const uint32_t tmem_o = tmem + lane_addr + L::kTmemO + t * D;
        // one-row-per-thread view of the same lane quarter, for the epilogue
        const uint32_t tmem_o_rows = tmem + (static_cast<uint32_t>(32 * q) << 16) + L::kTmemO + t * D;
        float* inv_l_sm = reinterpret_cast<float*>(smem + L::kInvLOff) + t * kBlockM;
        const float sl = p.scale_log2;
        uint32_t s_phase = 0, o_phase = 0, pair_phase = 0;
        uint32_t units = 0;  // units this warp has finished (for the staging tile's turn)
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
            const int row0 = tile_row0 + rr0;                 // global rows of r0 and r1
            const int row1 = row0 + 8;
            float m_run[2] = {-INFINITY, -INFINITY};  // running max per row, log2 units
            float l_run[2] = {0.f, 0.f};              // partial (this thread's columns) fp32 sums
            float lb_run[2] = {0.f, 0.f};             // the same over the bf16-rounded values

            for (int j = 0; j < nt; ++j) {
                ok = __all_sync(0xffffffffu, wait_bar(sync, s_full(t), s_phase));
                if (!ok) break;
                s_phase ^= 1;
                ptx::tc_fence_after_sync();

                const int key0 = j * kBlockN;
                const bool need_mask = (key0 + kBlockN > p.n) || (kCausal && key0 + kBlockN - 1 > tile_row0);
                const float slv = need_mask ? 1.f : sl;  // masked blocks are pre-scaled
                // Scores of this block into registers (masked keys to -inf,
                // scaled to log2 units, whatever the sign of the scale).
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
                // Exact row max (in log2 units), completed across the quad.
                auto block_max = [&](float (&mx)[2]) {
                    if (slv >= 0.f)
                        quad_row_extreme<true>(s, mx);
                    else
                        quad_row_extreme<false>(s, mx);
                    mx[0] *= slv;
                    mx[1] *= slv;
                };
                // p = 2^(s * slv - m): packed bf16 pairs, pk[2k] for r0 and
                // pk[2k + 1] for r1 in chunk k (the .16x128b store order), and
                // this thread's share of both row sums.
                uint32_t pk[32];
                float a[2][2], b[2][2];
                // chunks [k0, k1) of the block; a and b accumulate
                auto exponentiate_chunks = [&](const float (&neg_m)[2], int k0, int k1) {
#pragma unroll
                    for (int k = k0; k < k1; ++k) {
#pragma unroll
                        for (int r = 0; r < 2; ++r) {
                            float x0, x1, p0, p1;
                            ptx::fma2(x0, x1, s[4 * k + 2 * r], s[4 * k + 2 * r + 1], slv, slv, neg_m[r], neg_m[r]);
                            p0 = ptx::ex2(x0);
                            p1 = ptx::ex2(x1);
                            const uint32_t v = ptx::pack_bf16x2(p0, p1);
                            pk[2 * k + r] = v;
                            ptx::add2(a[r][0], a[r][1], a[r][0], a[r][1], p0, p1);
                            ptx::add_bf16x2_to_f32(b[r][0], b[r][1], v);
                        }
                    }
                };
                auto exponentiate = [&](const float (&neg_m)[2]) {
#pragma unroll
                    for (int r = 0; r < 2; ++r) a[r][0] = a[r][1] = b[r][0] = b[r][1] = 0.f;
                    exponentiate_chunks(neg_m, 0, 16);
                };
                auto neg_of = [](float m) { return (m == -INFINITY) ? 0.f : -m; };

                // Online softmax.  The first block of a unit sets the running
                // max exactly.  Later blocks exponentiate against the running
                // max as it stands and only check that no value exceeds
                // kStaleMaxBound (a value above it makes this thread's share of
                // a row sum exceed it); when one does -- the scores grew far past
                // everything seen so far -- the block is redone against its
                // exact max and O and l are rescaled.  O and l always share the
                // same m, so the result does not depend on how stale m is.
                // Causal instantiation, unmasked later blocks: the second
                // half of the block's columns loads while the first half is
                // exponentiated (no TMEM store is issued in between).  The
                // non-causal instantiation keeps one load at the top: with the
                // split the compiler spills there and it measured slower.
                if constexpr (!kCausal) load_scores();
                float alpha[2] = {1.f, 1.f};
                bool rescale_o = false;
                if (j == 0) {
                    if constexpr (kCausal) load_scores();
                    float mx[2];
                    block_max(mx);
                    m_run[0] = mx[0];
                    m_run[1] = mx[1];
                    const float nm[2] = {neg_of(m_run[0]), neg_of(m_run[1])};
                    exponentiate(nm);
                } else {
                    const float nm[2] = {neg_of(m_run[0]), neg_of(m_run[1])};
                    if (!kCausal || need_mask) {
                        if constexpr (kCausal) load_scores();
                        exponentiate(nm);
                    } else {
                        uint32_t(&lo)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[0]);
                        uint32_t(&hi)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[32]);
                        ptx::tmem_ld16x256b_x8_wait(tmem_s, lo);
                        ptx::tmem_ld16x256b_x8(tmem_s + 64, hi);
#pragma unroll
                        for (int r = 0; r < 2; ++r) a[r][0] = a[r][1] = b[r][0] = b[r][1] = 0.f;
                        exponentiate_chunks(nm, 0, 8);
                        ptx::tmem_wait_ld(hi);
                        exponentiate_chunks(nm, 8, 16);
                    }
                    const bool big = (a[0][0] + a[0][1] > kStaleMaxBound) || (a[1][0] + a[1][1] > kStaleMaxBound);
                    if (__any_sync(0xffffffffu, big)) {
                        load_scores();  // P has not been stored: S is still in TMEM
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

                // Rescale these rows of O_t.  S_t(j) being complete means every
                // earlier MMA (PV_t(j-1) included) is complete, so O_t is stable.
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
                // Every lane's P is in TMEM (its own wait and fence), the warp
                // meets, and one lane arrives: 8 arrivals per block instead
                // of 256 on the barrier the MMA warp is waiting on.
                ptx::tmem_st_wait();
                ptx::tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(p_full(t));
            }
            if (!ok) break;

            // Epilogue.  Row sums are complete once added across the quad.
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 1);
                l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 2);
                lb_run[r] += __shfl_xor_sync(0xffffffffu, lb_run[r], 1);
                lb_run[r] += __shfl_xor_sync(0xffffffffu, lb_run[r], 2);
            }
            ok = __all_sync(0xffffffffu, wait_bar(sync, o_full(t), o_phase));
            if (!ok) break;
            o_phase ^= 1;
            ptx::tc_fence_after_sync();
            if (qc == 0) {
                inv_l_sm[rr0] = 1.f / lb_run[0];
                inv_l_sm[rr0 + 8] = 1.f / lb_run[1];
                // lse in natural log, written once per row
                const float mu0 = (m_run[0] == -INFINITY) ? 0.f : m_run[0];
                const float mu1 = (m_run[1] == -INFINITY) ? 0.f : m_run[1];
                if (row0 < p.n) p.lse[static_cast<int64_t>(w.bh) * p.n + row0] = (mu0 + log2f(l_run[0])) * 0.69314718055994531f;
                if (row1 < p.n) p.lse[static_cast<int64_t>(w.bh) * p.n + row1] = (mu1 + log2f(l_run[1])) * 0.69314718055994531f;
            }
            // both warps of the lane quarter have published their rows' 1/l
            ptx::mbar_arrive(pair_bar(t, q));
            ok = __all_sync(0xffffffffu, wait_bar(sync, pair_bar(t, q), pair_phase));
            if (!ok) break;
            pair_phase ^= 1;
            // O = O_acc / l, written once: this warp converts columns
            // [D/2 h, D/2 (h+1)) of the quarter's 32 rows (one row per thread)
            // into the staging tile, laid out as the TMA store's 128-byte-
            // swizzled box (64-column panels; 16-byte chunk c of row r at
            // chunk position c ^ (r % 8)); the epilogue warp stores it.
            // Turn of the staging tile: tile 0's unit k follows tile 1's unit
            // k - 1, tile 1's follows tile 0's of the same unit.
            if (units > 0 || t == 1) {
                const uint32_t turn = 2 * units + static_cast<uint32_t>(t) - 1;
                ok = __all_sync(0xffffffffu, wait_bar(sync, stage_free, turn & 1));
                if (!ok) break;
            }
            const int rloc = 32 * q + lane;  // row in the tile
            const float inv_l = inv_l_sm[rloc];
            uint8_t* srow = smem + L::kStageOff + ((D / 2) * h / 64) * L::kPanelBytes + rloc * 128;
            const int chunk0 = ((D / 2) * h % 64) / 8;  // first 16-byte chunk of this warp's columns
#pragma unroll
            for (int c0 = 0; c0 < D / 2; c0 += 32) {
                uint32_t acc[32];
                ptx::tmem_ld32_wait(tmem_o_rows + (D / 2) * h + c0, acc);
                uint32_t packed[16];
#pragma unroll
                for (int c = 0; c < 32; c += 2)
                    packed[c >> 1] = ptx::pack_bf16x2(__uint_as_float(acc[c]) * inv_l,
                                                      __uint_as_float(acc[c + 1]) * inv_l);
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const int chunk = chunk0 + c0 / 8 + v;
                    *reinterpret_cast<uint4*>(srow + ((chunk ^ (rloc & 7)) << 4)) =
                        make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
                }
            }
            if (warp == 8 * t && lane == 0) {
                stage_coord[2 * t] = w.bh;
                stage_coord[2 * t + 1] = tile_row0;
            }
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before_sync();
            ptx::mbar_arrive(stage_full(t));
            ++units;
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
    clock_end(p, smem + L::kClockOff);
}

}  // namespace tc
}  // namespace fa
