// fa_api.cu -- the C ABI (include/fa.h): argument checks, kernel choice,
// TMA tensor-map encoding, persistent-grid sizing and launch on the caller's
// stream.  All compute runs in the kernels of fa_fwd_tc.cuh (bf16, tensor
// cores), fa_fwd_fp8_tc.cuh (E4M3, tensor cores), fa_fwd_simt.cuh (fp32,
// CUDA cores) and the decode, backward and merge kernels.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <functional>
#include <map>
#include <mutex>
#include <queue>
#include <tuple>
#include <vector>
#include <utility>
#include <string>

#include "fa.h"
#include "fa_testing.h"
#include "fa_bwd_tc.cuh"
#include "fa_decode.cuh"
#include "fa_decode_mma.cuh"
#include "fa_merge.cuh"
#include "fa_fwd_fp8_tc.cuh"
#include "fa_fwd_simt.cuh"
#include "fa_fwd_tc.cuh"
#include "fa_fwd_tc1.cuh"

namespace {

thread_local std::string g_last_error;

int fail(int code, const std::string& msg) {
    g_last_error = msg;
    return code;
}

int cuda_fail(cudaError_t e, const char* what) {
    return fail(FA_ERR_CUDA, std::string(what) + ": " + cudaGetErrorName(e) + " (" +
                                 cudaGetErrorString(e) + ")");
}

// Per-device state created on the first call that runs on that device and
// kept until process exit: a small device workspace holding the status word
// written by kernels that give up on a bounded wait, the forward kernels'
// clock record (SM cycles, timer nanoseconds, CTAs), followed by the work
// queues of the persistent kernel (two counters each, returned to zero by the
// last CTA of every launch); the SM count for the persistent grid; and
// whether the kernels' shared memory limits were raised.  Successive launches
// take successive queues, so launches in flight at the same time (on
// different streams) use different counters unless more than kQueues of them
// are in flight at once.
constexpr int kQueues = 1024;
constexpr size_t kClockOffset = 16;  // three 64-bit counters
constexpr size_t kQueueOffset = 48;
constexpr size_t kWorkspaceBytes = kQueueOffset + kQueues * 2 * sizeof(unsigned);

struct DeviceState {
    bool ready = false;
    int* status = nullptr;
    unsigned long long* clock = nullptr;
    unsigned* queues = nullptr;
    std::atomic<unsigned> next_queue{0};
    int sm_count = 0;
    int cc_major = 0;
    bool smem_raised[4] = {false, false, false, false};
    bool tile_smem_raised[4] = {false, false, false, false};
    bool decode_smem_raised[8] = {false, false, false, false, false, false, false, false};
    bool bwd_smem_raised[8] = {false, false, false, false, false, false, false, false};
    bool fp8_smem_raised[2] = {false, false};
    bool decode_mma_smem_raised[2] = {false, false};
};

constexpr int kMaxDevices = 64;
// set by fa_test_skip_one_arrival; consumed by the next bf16 launch of fa_fwd
std::atomic<int> g_skip_one_arrival{0};
// set by fa_test_force_forward_kernel: 0 by problem size, 1 two-tile, 2 one-tile
std::atomic<int> g_force_forward_kernel{0};
std::mutex g_mu;
DeviceState g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int device_state(DeviceState** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(FA_ERR_UNSUPPORTED, "device index out of range");
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceState& s = g_dev[dev];
    if (!s.ready) {
        if ((e = cudaDeviceGetAttribute(&s.sm_count, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return cuda_fail(e, "cudaDeviceGetAttribute(SM count)");
        if ((e = cudaDeviceGetAttribute(&s.cc_major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess)
            return cuda_fail(e, "cudaDeviceGetAttribute(compute capability)");
        if (!g_encode) {
            cudaDriverEntryPointQueryResult q;
            void* fn = nullptr;
            e = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q);
            if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
                return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled entry point not available");
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
        }
        void* ws = nullptr;
        if ((e = cudaMalloc(&ws, kWorkspaceBytes)) != cudaSuccess) return cuda_fail(e, "cudaMalloc(workspace)");
        if ((e = cudaMemset(ws, 0, kWorkspaceBytes)) != cudaSuccess) return cuda_fail(e, "cudaMemset(workspace)");
        s.status = static_cast<int*>(ws);
        s.clock = reinterpret_cast<unsigned long long*>(static_cast<char*>(ws) + kClockOffset);
        s.queues = reinterpret_cast<unsigned*>(static_cast<char*>(ws) + kQueueOffset);
        s.ready = true;
    }
    *out = &s;
    return FA_OK;
}

// Launch with programmatic stream serialization: the kernel's CTAs may start
// (shared memory, barriers, tensor memory) while the previous kernel of the
// stream finishes; the kernel waits for it (griddepcontrol.wait) before it
// touches global memory.
template <typename... Params, typename... Args>
cudaError_t launch_overlapped(void (*kernel)(Params...), int grid, int threads, int smem, cudaStream_t stream,
                              Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(static_cast<unsigned>(threads));
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

// 3-D view (d, N, B*H) of a [B*H][N][d] bf16 tensor, boxes of 64 x rows x 1
// (rows = 128 unless given) with 128-byte swizzle; rows past N read as zeros.
int encode_tile_map(CUtensorMap* map, const void* ptr, int64_t bh, int64_t n, int64_t d,
                    int rows = fa::tc::kBlockM) {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(n), static_cast<cuuint64_t>(bh)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d * 2), static_cast<cuuint64_t>(n * d * 2)};
    cuuint32_t box[3] = {64, static_cast<cuuint32_t>(rows), 1};
    cuuint32_t elem[3] = {1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
                          elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled failed with CUresult " + std::to_string(r));
    return FA_OK;
}

template <int D, bool kCausal>
int launch_bf16(DeviceState* st, int slot, const void* q, const void* k, const void* v, void* o, float* lse,
                int64_t bh, int64_t n, float scale, cudaStream_t stream) {
    using L = fa::tc::Layout<D>;
    auto kernel = fa::tc::fa_fwd_bf16_kernel<D, kCausal>;
    if (!st->smem_raised[slot]) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmemBytes);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(max dynamic shared memory)");
        std::lock_guard<std::mutex> lock(g_mu);
        st->smem_raised[slot] = true;
    }
    CUtensorMap tq, tk, tv, to;
    int rc;
    if ((rc = encode_tile_map(&tq, q, bh, n, D)) != FA_OK) return rc;
    if ((rc = encode_tile_map(&tk, k, bh, n, D)) != FA_OK) return rc;
    if ((rc = encode_tile_map(&tv, v, bh, n, D)) != FA_OK) return rc;
    if ((rc = encode_tile_map(&to, o, bh, n, D)) != FA_OK) return rc;

    fa::tc::Params p;
    p.o = static_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.status = st->status;
    p.sched = st->queues + 2 * (st->next_queue.fetch_add(1, std::memory_order_relaxed) % kQueues);
    p.bh = static_cast<int>(bh);
    p.n = static_cast<int>(n);
    p.num_qblocks = static_cast<int>((n + fa::tc::kUnitRows - 1) / fa::tc::kUnitRows);
    p.num_kblocks = static_cast<int>((n + fa::tc::kBlockN - 1) / fa::tc::kBlockN);
    p.num_units = p.bh * p.num_qblocks;
    p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    p.skip_one_arrival = g_skip_one_arrival.exchange(0);
    p.clock = st->clock;
    const int grid = p.num_units < st->sm_count ? p.num_units : st->sm_count;
    cudaError_t e = launch_overlapped(kernel, grid, fa::tc::kThreads, L::kSmemBytes, stream, tq, tk, tv, to, p);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "launch of the bf16 attention kernel");
    return FA_OK;
}

// The one-tile kernel (fa_fwd_tc1.cuh): 128-row units, one CTA per unit up
// to the SM count.
template <int D, bool kCausal>
int launch_bf16_tile(DeviceState* st, int slot, const void* q, const void* k, const void* v, void* o, float* lse,
                     int64_t bh, int64_t n, float scale, cudaStream_t stream) {
    using L = fa::tc1::Layout<D>;
    auto kernel = fa::tc1::fa_fwd_bf16_tile_kernel<D, kCausal>;
    if (!st->tile_smem_raised[slot]) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmemBytes);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(max dynamic shared memory)");
        std::lock_guard<std::mutex> lock(g_mu);
        st->tile_smem_raised[slot] = true;
    }
    CUtensorMap tq, tk, tv;
    int rc;
    if ((rc = encode_tile_map(&tq, q, bh, n, D)) != FA_OK) return rc;
    if ((rc = encode_tile_map(&tk, k, bh, n, D)) != FA_OK) return rc;
    if ((rc = encode_tile_map(&tv, v, bh, n, D)) != FA_OK) return rc;

    fa::tc::Params p;
    p.o = static_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.status = st->status;
    p.sched = st->queues + 2 * (st->next_queue.fetch_add(1, std::memory_order_relaxed) % kQueues);
    p.bh = static_cast<int>(bh);
    p.n = static_cast<int>(n);
    p.num_qblocks = static_cast<int>((n + fa::tc::kBlockM - 1) / fa::tc::kBlockM);  // 128-row units
    p.num_kblocks = static_cast<int>((n + fa::tc::kBlockN - 1) / fa::tc::kBlockN);
    p.num_units = p.bh * p.num_qblocks;
    p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    p.skip_one_arrival = g_skip_one_arrival.exchange(0);
    p.clock = st->clock;
    const int grid = p.num_units < st->sm_count ? p.num_units : st->sm_count;
    cudaError_t e = launch_overlapped(kernel, grid, fa::tc1::kThreads, L::kSmemBytes, stream, tq, tk, tv, p);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "launch of the one-tile bf16 attention kernel");
    return FA_OK;
}

template <int D, bool kCausal>
int launch_f32(const void* q, const void* k, const void* v, void* o, float* lse, int64_t bh, int64_t n,
               float scale, cudaStream_t stream) {
    fa::simt::Params p;
    p.q = static_cast<const float*>(q);
    p.k = static_cast<const float*>(k);
    p.v = static_cast<const float*>(v);
    p.o = static_cast<float*>(o);
    p.lse = lse;
    p.n = static_cast<int>(n);
    p.scale = scale;
    dim3 grid(static_cast<unsigned>((n + fa::simt::kRows - 1) / fa::simt::kRows), static_cast<unsigned>(bh));
    fa::simt::fa_fwd_f32_kernel<D, kCausal><<<grid, fa::simt::kThreads, 0, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "launch of the fp32 attention kernel");
    return FA_OK;
}

// Argument checks shared by the entry points; all run before any CUDA call.
struct Sizes {
    int64_t bh = 0;
    int64_t elem = 0;
    size_t tensor_bytes = 0;
    size_t lse_bytes = 0;
};

int check_args(const void* q, const void* k, const void* v, const void* o, const float* lse, int64_t B,
               int64_t H, int64_t N, int64_t d, float scale, int dtype, bool device_pointers, Sizes* z) {
    if (!q || !k || !v || !o || !lse) return fail(FA_ERR_INVALID_ARGUMENT, "null pointer argument");
    if (B < 1 || H < 1 || N < 1 || d < 1) return fail(FA_ERR_INVALID_ARGUMENT, "B, H, N and d must be >= 1");
    if (dtype != FA_DTYPE_F32 && dtype != FA_DTYPE_BF16) return fail(FA_ERR_INVALID_ARGUMENT, "unknown dtype");
    if (!std::isfinite(scale)) return fail(FA_ERR_INVALID_ARGUMENT, "scale must be finite");
    if (d != 64 && d != 128) return fail(FA_ERR_UNSUPPORTED, "head dim must be 64 or 128");
    if (B > INT_MAX / H) return fail(FA_ERR_INVALID_ARGUMENT, "B * H too large");
    const int64_t bh = B * H;
    if (N > (int64_t{1} << 30)) return fail(FA_ERR_INVALID_ARGUMENT, "N too large (max 2^30)");
    const int64_t units = bh * ((N + 255) / 256);
    if (units > INT_MAX) return fail(FA_ERR_INVALID_ARGUMENT, "B * H * N too large");
    const int64_t elem = dtype == FA_DTYPE_BF16 ? 2 : 4;
    if (bh > (int64_t{1} << 62) / (N * d * elem)) return fail(FA_ERR_INVALID_ARGUMENT, "tensor size overflows");
    const size_t tensor_bytes = static_cast<size_t>(bh * N * d * elem);
    const size_t lse_bytes = static_cast<size_t>(bh * N * 4);
    auto misaligned = [](const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) != 0; };
    if (device_pointers) {
        if (misaligned(q, 16) || misaligned(k, 16) || misaligned(v, 16) || misaligned(o, 16))
            return fail(FA_ERR_INVALID_ARGUMENT, "q, k, v and o must be 16-byte aligned");
        if (misaligned(lse, 4)) return fail(FA_ERR_INVALID_ARGUMENT, "lse must be 4-byte aligned");
    }
    if (overlaps(o, tensor_bytes, q, tensor_bytes) || overlaps(o, tensor_bytes, k, tensor_bytes) ||
        overlaps(o, tensor_bytes, v, tensor_bytes) || overlaps(o, tensor_bytes, lse, lse_bytes))
        return fail(FA_ERR_INVALID_ARGUMENT, "o overlaps another argument");
    if (overlaps(lse, lse_bytes, q, tensor_bytes) || overlaps(lse, lse_bytes, k, tensor_bytes) ||
        overlaps(lse, lse_bytes, v, tensor_bytes))
        return fail(FA_ERR_INVALID_ARGUMENT, "lse overlaps another argument");
    z->bh = bh;
    z->elem = elem;
    z->tensor_bytes = tensor_bytes;
    z->lse_bytes = lse_bytes;
    return FA_OK;
}

// Which bf16 kernel runs a problem.  Both kernels take their work units
// from a queue in the same order (groups of kHeadGroup heads; under the causal
// mask each group's heaviest query blocks first) and every CTA takes the next
// unit when it is free, so a launch lasts as long as the busiest CTA of that
// list schedule.  A unit costs its KV blocks times the cycles one block takes:
// ~1886 for the one-tile kernel's 128 rows, ~3245 for the two-tile kernel's
// 256 rows (clock64 traces of both kernels in steady state).  The one-tile
// kernel is picked when its schedule is the shorter: always when every tile
// has its own SM, never beyond 8 tiles per SM (there its doubled K/V reads
// and per-block cost always lose), by simulating both schedules in between
// (cached per shape).  Measured on 64 shapes (B, H, N in 1..4, 4..64,
// 1K..16K, d 64 and 128, both masks) this picks the faster kernel in 62.
constexpr double kCyclesPerBlockOneTile = 1886.0;
constexpr double kCyclesPerBlockPairTwoTile = 3245.0;

double list_schedule_cycles(int64_t bh, int64_t n, bool causal, bool one_tile, int sms) {
    const int64_t nb = (n + fa::tc::kBlockN - 1) / fa::tc::kBlockN;
    const int64_t rows = one_tile ? fa::tc::kBlockM : fa::tc::kUnitRows;
    const int64_t nq = (n + rows - 1) / rows;
    const double c = one_tile ? kCyclesPerBlockOneTile : kCyclesPerBlockPairTwoTile;
    const int64_t units = bh * nq;
    const int64_t ctas = units < sms ? units : sms;
    std::priority_queue<double, std::vector<double>, std::greater<double>> busy;
    for (int64_t i = 0; i < ctas; ++i) busy.push(0.0);
    double end = 0.0;
    for (int64_t g0 = 0; g0 < bh; g0 += fa::tc::kHeadGroup) {
        const int64_t hg = (bh - g0 < fa::tc::kHeadGroup) ? bh - g0 : fa::tc::kHeadGroup;
        for (int64_t qi = 0; qi < nq; ++qi) {
            const int64_t qb = causal ? nq - 1 - qi : qi;
            int64_t blocks = nb;
            if (causal) {
                const int64_t last = one_tile ? qb + 1 : 2 * qb + 2;  // through the diagonal block
                blocks = last < nb ? last : nb;
            }
            for (int64_t h = 0; h < hg; ++h) {
                const double t = busy.top() + c * static_cast<double>(blocks);
                busy.pop();
                busy.push(t);
                end = t > end ? t : end;
            }
        }
    }
    return end;
}

bool one_tile_is_faster(int64_t bh, int64_t n, bool causal, int sms) {
    const int64_t tiles = bh * ((n + fa::tc::kBlockM - 1) / fa::tc::kBlockM);
    if (tiles <= sms) return true;
    if (tiles > 8 * static_cast<int64_t>(sms)) return false;
    static std::mutex mu;
    static std::map<std::tuple<int64_t, int64_t, bool, int>, bool> cache;
    const auto key = std::make_tuple(bh, n, causal, sms);
    {
        std::lock_guard<std::mutex> lock(mu);
        auto it = cache.find(key);
        if (it != cache.end()) return it->second;
    }
    const bool one = list_schedule_cycles(bh, n, causal, true, sms) < list_schedule_cycles(bh, n, causal, false, sms);
    std::lock_guard<std::mutex> lock(mu);
    if (cache.size() < 4096) cache.emplace(key, one);
    return one;
}

// Kernel choice and launch on `s` for bh heads of N rows (device pointers).
int dispatch(DeviceState* st, const void* q, const void* k, const void* v, void* o, float* lse, int64_t bh,
             int64_t N, int64_t d, float scale, bool c, int dtype, cudaStream_t s) {
    if (dtype == FA_DTYPE_BF16) {
        if (st->cc_major != 10)
            return fail(FA_ERR_UNSUPPORTED, "the bf16 kernel needs an sm_100 (B200-class) GPU");
        const int force = g_force_forward_kernel.load();
        if (force == 2 || (force == 0 && one_tile_is_faster(bh, N, c, st->sm_count))) {
            if (d == 128) return c ? launch_bf16_tile<128, true>(st, 0, q, k, v, o, lse, bh, N, scale, s)
                                   : launch_bf16_tile<128, false>(st, 1, q, k, v, o, lse, bh, N, scale, s);
            return c ? launch_bf16_tile<64, true>(st, 2, q, k, v, o, lse, bh, N, scale, s)
                     : launch_bf16_tile<64, false>(st, 3, q, k, v, o, lse, bh, N, scale, s);
        }
        if (d == 128) return c ? launch_bf16<128, true>(st, 0, q, k, v, o, lse, bh, N, scale, s)
                               : launch_bf16<128, false>(st, 1, q, k, v, o, lse, bh, N, scale, s);
        return c ? launch_bf16<64, true>(st, 2, q, k, v, o, lse, bh, N, scale, s)
                 : launch_bf16<64, false>(st, 3, q, k, v, o, lse, bh, N, scale, s);
    }
    if (d == 128) return c ? launch_f32<128, true>(q, k, v, o, lse, bh, N, scale, s)
                           : launch_f32<128, false>(q, k, v, o, lse, bh, N, scale, s);
    return c ? launch_f32<64, true>(q, k, v, o, lse, bh, N, scale, s)
             : launch_f32<64, false>(q, k, v, o, lse, bh, N, scale, s);
}

}  // namespace

extern "C" {

int fa_test_skip_one_arrival(void) {
    g_skip_one_arrival.store(1);
    return FA_OK;
}

int fa_fwd_kernel_choice(int64_t B, int64_t H, int64_t N, int64_t d, int causal, int dtype, int sm_count,
                         int* kernel) {
    g_last_error.clear();
    if (!kernel) return fail(FA_ERR_INVALID_ARGUMENT, "kernel is null");
    if (B < 1 || H < 1 || N < 1) return fail(FA_ERR_INVALID_ARGUMENT, "B, H and N must be >= 1");
    if (dtype != FA_DTYPE_F32 && dtype != FA_DTYPE_BF16) return fail(FA_ERR_INVALID_ARGUMENT, "unknown dtype");
    if (d != 64 && d != 128) return fail(FA_ERR_UNSUPPORTED, "head dim must be 64 or 128");
    if (B > INT_MAX / H) return fail(FA_ERR_INVALID_ARGUMENT, "B * H too large");
    if (N > (int64_t{1} << 30)) return fail(FA_ERR_INVALID_ARGUMENT, "N too large (max 2^30)");
    if (dtype == FA_DTYPE_F32) {
        *kernel = FA_KERNEL_F32;
        return FA_OK;
    }
    if (sm_count < 1) {
        DeviceState* st = nullptr;
        int rc = device_state(&st);
        if (rc != FA_OK) return rc;
        sm_count = st->sm_count;
    }
    *kernel = one_tile_is_faster(B * H, N, causal != 0, sm_count) ? FA_KERNEL_BF16_ONE_TILE : FA_KERNEL_BF16_TWO_TILE;
    return FA_OK;
}

int fa_test_force_forward_kernel(int which) {
    g_last_error.clear();
    if (which < 0 || which > 2) return fail(FA_ERR_INVALID_ARGUMENT, "which must be 0, 1 or 2");
    g_force_forward_kernel.store(which);
    return FA_OK;
}

int fa_version(void) { return FA_VERSION_MAJOR * 10000 + FA_VERSION_MINOR * 100 + FA_VERSION_PATCH; }

const char* fa_status_string(int status) {
    switch (status) {
        case FA_OK: return "FA_OK: success";
        case FA_ERR_INVALID_ARGUMENT: return "FA_ERR_INVALID_ARGUMENT: bad pointer, size, alignment, aliasing, dtype or scale";
        case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED: well-formed request this library does not implement";
        case FA_ERR_CUDA: return "FA_ERR_CUDA: a CUDA call failed";
        case FA_ERR_DEVICE_TIMEOUT: return "FA_ERR_DEVICE_TIMEOUT: a kernel gave up on a bounded wait; outputs invalid";
        default: return "unknown fa status code";
    }
}

const char* fa_last_error(void) { return g_last_error.c_str(); }

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t H, int64_t N,
           int64_t d, float scale, int causal, int dtype, void* stream) {
    g_last_error.clear();
    Sizes z;
    int rc = check_args(q, k, v, o, lse, B, H, N, d, scale, dtype, true, &z);
    if (rc != FA_OK) return rc;
    DeviceState* st = nullptr;
    if ((rc = device_state(&st)) != FA_OK) return rc;
    return dispatch(st, q, k, v, o, lse, z.bh, N, d, scale, causal != 0, dtype, static_cast<cudaStream_t>(stream));
}

int fa_check_device_status(void* stream) {
    g_last_error.clear();
    DeviceState* st = nullptr;
    int rc = device_state(&st);
    if (rc != FA_OK) return rc;
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    int h = 0;
    if ((e = cudaMemcpy(&h, st->status, sizeof(int), cudaMemcpyDeviceToHost)) != cudaSuccess)
        return cuda_fail(e, "cudaMemcpy(status word)");
    if (h != 0) {
        if ((e = cudaMemset(st->status, 0, sizeof(int))) != cudaSuccess) return cuda_fail(e, "cudaMemset(status word)");
        return fail(FA_ERR_DEVICE_TIMEOUT, "a kernel gave up on a bounded wait");
    }
    return FA_OK;
}

int fa_clock_record(void* stream, int reset, int64_t* out) {
    g_last_error.clear();
    if (!out) return fail(FA_ERR_INVALID_ARGUMENT, "out is null");
    DeviceState* st = nullptr;
    int rc = device_state(&st);
    if (rc != FA_OK) return rc;
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    unsigned long long h[3] = {0, 0, 0};
    if ((e = cudaMemcpy(h, st->clock, sizeof(h), cudaMemcpyDeviceToHost)) != cudaSuccess)
        return cuda_fail(e, "cudaMemcpy(clock record)");
    for (int i = 0; i < 3; ++i) out[i] = static_cast<int64_t>(h[i]);
    if (reset && (e = cudaMemset(st->clock, 0, sizeof(h))) != cudaSuccess)
        return cuda_fail(e, "cudaMemset(clock record)");
    return FA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// fa_fwd_noalloc: the same forward for callers that must not allocate device
// memory.  fa_fwd allocates a small workspace (device status word and
// work-queue counters) with cudaMalloc on its first call on each device; some
// callers cannot let a library do that -- a serving process that has already
// reserved the whole GPU memory for its own pool, code that runs inside an
// allocator's hooks, or deployments with strict per-library memory budgets.
// This entry point keeps that scratch in a fixed, file-scope device array
// instead and calls no allocating routine.
namespace {

// 256 bytes of scratch, loaded with the library on every GPU it runs on and
// kept until the process exits (zero when the library is loaded).  Word 0:
// device status (a kernel that gave up on a bounded wait sets it; it stays set
// until fa_noalloc_check_status reads it); words 4 and 5: the persistent
// kernel's work queue (next unit, CTAs finished), cleared before every launch.
// The rest is unused headroom.
constexpr int kNoAllocScratchWords = 64;
constexpr int kNoAllocStatusWord = 0;
constexpr int kNoAllocQueueWord = 4;
constexpr int kNoAllocQueueWords = 2;
static __device__ __align__(256) unsigned g_noalloc_scratch[kNoAllocScratchWords];
static_assert(kNoAllocQueueWord + kNoAllocQueueWords <= kNoAllocScratchWords, "no-alloc scratch too small");

struct NoAllocDevice {
    bool ready = false;
    unsigned* scratch = nullptr;  // device address of g_noalloc_scratch on this device
    int sm_count = 0;
    int cc_major = 0;
    bool smem_raised[4] = {false, false, false, false};
    bool tile_smem_raised[4] = {false, false, false, false};
};
NoAllocDevice g_noalloc_dev[kMaxDevices];

// First call on a device (with that device current): look up the scratch
// array's device address and the launch attributes.  Nothing is allocated.
int noalloc_setup(NoAllocDevice** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(FA_ERR_UNSUPPORTED, "device index out of range");
    std::lock_guard<std::mutex> lock(g_mu);
    NoAllocDevice& s = g_noalloc_dev[dev];
    if (!s.ready) {
        if ((e = cudaDeviceGetAttribute(&s.sm_count, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return cuda_fail(e, "cudaDeviceGetAttribute(SM count)");
        if ((e = cudaDeviceGetAttribute(&s.cc_major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess)
            return cuda_fail(e, "cudaDeviceGetAttribute(compute capability)");
        if (!g_encode) {
            cudaDriverEntryPointQueryResult q;
            void* fn = nullptr;
            e = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q);
            if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
                return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled entry point not available");
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
        }
        void* ptr = nullptr;
        if ((e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch)) != cudaSuccess)
            return cuda_fail(e, "cudaGetSymbolAddress(no-alloc scratch)");
        s.scratch = static_cast<unsigned*>(ptr);
        s.ready = true;
    }
    *out = &s;
    return FA_OK;
}

template <int D, bool kCausal>
int launch_bf16_noalloc(NoAllocDevice* st, int slot, const void* q, const void* k, const void* v, void* o,
                        float* lse, int64_t bh, int64_t n, float scale, cudaStream_t stream) {
    using L = fa::tc::Layout<D>;
    auto kernel = fa::tc::fa_fwd_bf16_kernel<D, kCausal>;
    if (!st->smem_raised[slot]) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmemBytes);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(max dynamic shared memory)");
        std::lock_guard<std::mutex> lock(g_mu);
        st->smem_raised[slot] = true;
    }
    CUtensorMap tq, tk, tv, to;
    int rc;
    if ((rc = encode_tile_map(&tq, q, bh, n, D)) != FA_OK) return rc;
    if ((rc = encode_tile_map(&tk, k, bh, n, D)) != FA_OK) return rc;
    if ((rc = encode_tile_map(&tv, v, bh, n, D)) != FA_OK) return rc;
    if ((rc = encode_tile_map(&to, o, bh, n, D)) != FA_OK) return rc;
    // The array keeps the previous call's contents: the queue counters must
    // start at zero, so clear them in stream order.  The status word is left
    // alone, so that a timeout stays visible until fa_noalloc_check_status.
    cudaError_t e = cudaMemsetAsync(st->scratch + kNoAllocQueueWord, 0, kNoAllocQueueWords * sizeof(unsigned), stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(no-alloc queue words)");

    fa::tc::Params p;
    p.o = static_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.status = reinterpret_cast<int*>(st->scratch + kNoAllocStatusWord);
    p.sched = st->scratch + kNoAllocQueueWord;
    p.bh = static_cast<int>(bh);
    p.n = static_cast<int>(n);
    p.num_qblocks = static_cast<int>((n + fa::tc::kUnitRows - 1) / fa::tc::kUnitRows);
    p.num_kblocks = static_cast<int>((n + fa::tc::kBlockN - 1) / fa::tc::kBlockN);
    p.num_units = p.bh * p.num_qblocks;
    p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    p.skip_one_arrival = g_skip_one_arrival.exchange(0);
    p.clock = nullptr;  // nothing of the shared workspace is touched here
    const int grid = p.num_units < st->sm_count ? p.num_units : st->sm_count;
    kernel<<<grid, fa::tc::kThreads, L::kSmemBytes, stream>>>(tq, tk, tv, to, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "launch of the bf16 attention kernel (no-alloc)");
    return FA_OK;
}

// The one-tile kernel with the no-alloc scratch (same queue and status words).
template <int D, bool kCausal>
int launch_bf16_tile_noalloc(NoAllocDevice* st, int slot, const void* q, const void* k, const void* v, void* o,
                             float* lse, int64_t bh, int64_t n, float scale, cudaStream_t stream) {
    using L = fa::tc1::Layout<D>;
    auto kernel = fa::tc1::fa_fwd_bf16_tile_kernel<D, kCausal>;
    if (!st->tile_smem_raised[slot]) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmemBytes);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(max dynamic shared memory)");
        std::lock_guard<std::mutex> lock(g_mu);
        st->tile_smem_raised[slot] = true;
    }
    CUtensorMap tq, tk, tv;
    int rc;
    if ((rc = encode_tile_map(&tq, q, bh, n, D)) != FA_OK) return rc;
    if ((rc = encode_tile_map(&tk, k, bh, n, D)) != FA_OK) return rc;
    if ((rc = encode_tile_map(&tv, v, bh, n, D)) != FA_OK) return rc;
    cudaError_t e = cudaMemsetAsync(st->scratch + kNoAllocQueueWord, 0, kNoAllocQueueWords * sizeof(unsigned), stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(no-alloc queue words)");

    fa::tc::Params p;
    p.o = static_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.status = reinterpret_cast<int*>(st->scratch + kNoAllocStatusWord);
    p.sched = st->scratch + kNoAllocQueueWord;
    p.bh = static_cast<int>(bh);
    p.n = static_cast<int>(n);
    p.num_qblocks = static_cast<int>((n + fa::tc::kBlockM - 1) / fa::tc::kBlockM);  // 128-row units
    p.num_kblocks = static_cast<int>((n + fa::tc::kBlockN - 1) / fa::tc::kBlockN);
    p.num_units = p.bh * p.num_qblocks;
    p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    p.skip_one_arrival = g_skip_one_arrival.exchange(0);
    p.clock = nullptr;
    const int grid = p.num_units < st->sm_count ? p.num_units : st->sm_count;
    kernel<<<grid, fa::tc1::kThreads, L::kSmemBytes, stream>>>(tq, tk, tv, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "launch of the one-tile bf16 attention kernel (no-alloc)");
    return FA_OK;
}

}  // namespace

extern "C" int fa_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B,
                              int64_t H, int64_t N, int64_t d, float scale, int causal, int dtype,
                              void* stream) {
    g_last_error.clear();
    // ---- the same argument checks as fa_fwd, before any CUDA call
    if (!q || !k || !v || !o || !lse) return fail(FA_ERR_INVALID_ARGUMENT, "null pointer argument");
    if (B < 1 || H < 1 || N < 1 || d < 1) return fail(FA_ERR_INVALID_ARGUMENT, "B, H, N and d must be >= 1");
    if (dtype != FA_DTYPE_F32 && dtype != FA_DTYPE_BF16) return fail(FA_ERR_INVALID_ARGUMENT, "unknown dtype");
    if (!std::isfinite(scale)) return fail(FA_ERR_INVALID_ARGUMENT, "scale must be finite");
    if (d != 64 && d != 128) return fail(FA_ERR_UNSUPPORTED, "head dim must be 64 or 128");
    if (B > INT_MAX / H) return fail(FA_ERR_INVALID_ARGUMENT, "B * H too large");
    const int64_t bh = B * H;
    if (N > (int64_t{1} << 30)) return fail(FA_ERR_INVALID_ARGUMENT, "N too large (max 2^30)");
    const int64_t units = bh * ((N + 255) / 256);
    if (units > INT_MAX) return fail(FA_ERR_INVALID_ARGUMENT, "B * H * N too large");
    const int64_t elem = dtype == FA_DTYPE_BF16 ? 2 : 4;
    if (bh > (int64_t{1} << 62) / (N * d * elem)) return fail(FA_ERR_INVALID_ARGUMENT, "tensor size overflows");
    const size_t tensor_bytes = static_cast<size_t>(bh * N * d * elem);
    const size_t lse_bytes = static_cast<size_t>(bh * N * 4);
    auto misaligned = [](const void* ptr, uintptr_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) != 0; };
    if (misaligned(q, 16) || misaligned(k, 16) || misaligned(v, 16) || misaligned(o, 16))
        return fail(FA_ERR_INVALID_ARGUMENT, "q, k, v and o must be 16-byte aligned");
    if (misaligned(lse, 4)) return fail(FA_ERR_INVALID_ARGUMENT, "lse must be 4-byte aligned");
    if (overlaps(o, tensor_bytes, q, tensor_bytes) || overlaps(o, tensor_bytes, k, tensor_bytes) ||
        overlaps(o, tensor_bytes, v, tensor_bytes) || overlaps(o, tensor_bytes, lse, lse_bytes))
        return fail(FA_ERR_INVALID_ARGUMENT, "o overlaps another argument");
    if (overlaps(lse, lse_bytes, q, tensor_bytes) || overlaps(lse, lse_bytes, k, tensor_bytes) ||
        overlaps(lse, lse_bytes, v, tensor_bytes))
        return fail(FA_ERR_INVALID_ARGUMENT, "lse overlaps another argument");

    // ---- set-up on the first call per device (no allocation) and dispatch
    NoAllocDevice* st = nullptr;
    int rc = noalloc_setup(&st);
    if (rc != FA_OK) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool c = causal != 0;
    if (dtype == FA_DTYPE_BF16) {
        if (st->cc_major != 10)
            return fail(FA_ERR_UNSUPPORTED, "the bf16 kernel needs an sm_100 (B200-class) GPU");
        // the one-tile kernel when every 128-row tile has its own SM (the choice
        // fa_fwd makes by a schedule simulation keeps host state; this rule
        // keeps none and agrees with it there)
        const int force = g_force_forward_kernel.load();
        const int64_t tiles = bh * ((N + fa::tc::kBlockM - 1) / fa::tc::kBlockM);
        if (force == 2 || (force == 0 && tiles <= st->sm_count)) {
            if (d == 128) return c ? launch_bf16_tile_noalloc<128, true>(st, 0, q, k, v, o, lse, bh, N, scale, s)
                                   : launch_bf16_tile_noalloc<128, false>(st, 1, q, k, v, o, lse, bh, N, scale, s);
            return c ? launch_bf16_tile_noalloc<64, true>(st, 2, q, k, v, o, lse, bh, N, scale, s)
                     : launch_bf16_tile_noalloc<64, false>(st, 3, q, k, v, o, lse, bh, N, scale, s);
        }
        if (d == 128) return c ? launch_bf16_noalloc<128, true>(st, 0, q, k, v, o, lse, bh, N, scale, s)
                               : launch_bf16_noalloc<128, false>(st, 1, q, k, v, o, lse, bh, N, scale, s);
        return c ? launch_bf16_noalloc<64, true>(st, 2, q, k, v, o, lse, bh, N, scale, s)
                 : launch_bf16_noalloc<64, false>(st, 3, q, k, v, o, lse, bh, N, scale, s);
    }
    // the fp32 kernel uses no scratch at all
    if (d == 128) return c ? launch_f32<128, true>(q, k, v, o, lse, bh, N, scale, s)
                           : launch_f32<128, false>(q, k, v, o, lse, bh, N, scale, s);
    return c ? launch_f32<64, true>(q, k, v, o, lse, bh, N, scale, s)
             : launch_f32<64, false>(q, k, v, o, lse, bh, N, scale, s);
}

extern "C" int fa_noalloc_check_status(void* stream) {
    g_last_error.clear();
    NoAllocDevice* st = nullptr;
    int rc = noalloc_setup(&st);
    if (rc != FA_OK) return rc;
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    unsigned h = 0;
    if ((e = cudaMemcpy(&h, st->scratch + kNoAllocStatusWord, sizeof(unsigned), cudaMemcpyDeviceToHost)) != cudaSuccess)
        return cuda_fail(e, "cudaMemcpy(no-alloc status word)");
    if (h != 0) {
        if ((e = cudaMemset(st->scratch + kNoAllocStatusWord, 0, sizeof(unsigned))) != cudaSuccess)
            return cuda_fail(e, "cudaMemset(no-alloc status word)");
        return fail(FA_ERR_DEVICE_TIMEOUT, "a kernel launched by fa_fwd_noalloc gave up on a bounded wait");
    }
    return FA_OK;
}

// ---------------------------------------------------------------------------
// fa_fwd_host: the forward on host buffers.  The heads are processed in
// chunks through three device staging buffers on three internal streams, so
// that the copy-in of one chunk, the kernel of the previous one and the
// copy-out of the one before run at the same time (host-to-device and
// device-to-host copies use separate copy engines).  For pinned host memory
// the whole call then costs about the longer of the two copy directions
// instead of their sum plus the kernel.
namespace {

constexpr int kPipeBuffers = 3;
constexpr int64_t kPipeChunks = 8;  // target number of chunks per call

struct HostPipe {
    bool ready = false;
    cudaStream_t s_in = nullptr, s_comp = nullptr, s_out = nullptr;
    cudaEvent_t ev_entry = nullptr, ev_done = nullptr;
    cudaEvent_t ev_in[kPipeBuffers] = {}, ev_comp[kPipeBuffers] = {}, ev_free[kPipeBuffers] = {};
    char* buf[kPipeBuffers] = {};
    size_t buf_bytes = 0;
    std::mutex mu;  // one call at a time enqueues on this device's pipeline
};
HostPipe g_pipe[kMaxDevices];

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int pipe_setup(HostPipe& pp) {
    if (pp.ready) return FA_OK;
    cudaError_t e;
    for (cudaStream_t* s : {&pp.s_in, &pp.s_comp, &pp.s_out})
        if ((e = cudaStreamCreateWithFlags(s, cudaStreamNonBlocking)) != cudaSuccess)
            return cuda_fail(e, "cudaStreamCreateWithFlags");
    if ((e = cudaEventCreateWithFlags(&pp.ev_entry, cudaEventDisableTiming)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&pp.ev_done, cudaEventDisableTiming)) != cudaSuccess)
        return cuda_fail(e, "cudaEventCreateWithFlags");
    for (int b = 0; b < kPipeBuffers; ++b)
        for (cudaEvent_t* ev : {&pp.ev_in[b], &pp.ev_comp[b], &pp.ev_free[b]})
            if ((e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming)) != cudaSuccess)
                return cuda_fail(e, "cudaEventCreateWithFlags");
    pp.ready = true;
    return FA_OK;
}

// Staging buffers of at least `bytes` each; growing waits for the pipeline
// to drain first, since queued work may still use the old buffers.
int pipe_reserve(HostPipe& pp, size_t bytes) {
    if (pp.buf_bytes >= bytes) return FA_OK;
    cudaError_t e;
    for (cudaStream_t s : {pp.s_in, pp.s_comp, pp.s_out})
        if ((e = cudaStreamSynchronize(s)) != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    for (int b = 0; b < kPipeBuffers; ++b) {
        if (pp.buf[b] && (e = cudaFree(pp.buf[b])) != cudaSuccess) return cuda_fail(e, "cudaFree(staging)");
        pp.buf[b] = nullptr;
    }
    pp.buf_bytes = 0;
    for (int b = 0; b < kPipeBuffers; ++b)
        if ((e = cudaMalloc(&pp.buf[b], bytes)) != cudaSuccess) return cuda_fail(e, "cudaMalloc(staging)");
    pp.buf_bytes = bytes;
    return FA_OK;
}

// Copy-in, kernel, copy-out over chunks of heads.  in_head / out_head: bytes
// of one head of q (k, v alike) and of o; launch(dq, dk, dv, do, dl, heads,
// stream) runs the kernel on a chunk's device copies.
template <typename Launch>
int host_pipeline(const void* q, const void* k, const void* v, void* o, float* lse, int64_t bh, int64_t N,
                  size_t in_head, size_t out_head, cudaStream_t caller, Launch&& launch) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    HostPipe& pp = g_pipe[dev];
    std::lock_guard<std::mutex> lock(pp.mu);
    int rc;
    if ((rc = pipe_setup(pp)) != FA_OK) return rc;

    const int64_t ch = (bh + kPipeChunks - 1) / kPipeChunks;  // heads per chunk
    const size_t head_lse = static_cast<size_t>(N * 4);
    const size_t t_in = round_up(ch * in_head, 256), t_out = round_up(ch * out_head, 256);
    const size_t l_bytes = round_up(ch * head_lse, 256);
    if ((rc = pipe_reserve(pp, 3 * t_in + t_out + l_bytes)) != FA_OK) return rc;

    auto ck = [&](cudaError_t err, const char* what) { return err == cudaSuccess ? FA_OK : cuda_fail(err, what); };
    if ((rc = ck(cudaEventRecord(pp.ev_entry, caller), "cudaEventRecord")) != FA_OK) return rc;
    if ((rc = ck(cudaStreamWaitEvent(pp.s_in, pp.ev_entry, 0), "cudaStreamWaitEvent")) != FA_OK) return rc;
    const char* hq = static_cast<const char*>(q);
    const char* hk = static_cast<const char*>(k);
    const char* hv = static_cast<const char*>(v);
    char* ho = static_cast<char*>(o);
    char* hl = reinterpret_cast<char*>(lse);
    const int64_t nchunks = (bh + ch - 1) / ch;
    for (int64_t i = 0; i < nchunks; ++i) {
        const int b = static_cast<int>(i % kPipeBuffers);
        const int64_t h0 = i * ch, hc = (h0 + ch <= bh) ? ch : bh - h0;
        const size_t off = static_cast<size_t>(h0) * in_head, nb = static_cast<size_t>(hc) * in_head;
        const size_t ooff = static_cast<size_t>(h0) * out_head, onb = static_cast<size_t>(hc) * out_head;
        const size_t loff = static_cast<size_t>(h0) * head_lse, lnb = static_cast<size_t>(hc) * head_lse;
        char* dq = pp.buf[b];
        char* dk = dq + t_in;
        char* dv = dk + t_in;
        char* dout = dv + t_in;
        float* dl = reinterpret_cast<float*>(dout + t_out);
        // copy-in once the buffer's previous chunk (of this call or an earlier
        // one) has been copied out; an event never recorded is no wait
        if ((rc = ck(cudaStreamWaitEvent(pp.s_in, pp.ev_free[b], 0), "cudaStreamWaitEvent")) != FA_OK) return rc;
        if ((rc = ck(cudaMemcpyAsync(dq, hq + off, nb, cudaMemcpyDefault, pp.s_in), "cudaMemcpyAsync(q)")) != FA_OK ||
            (rc = ck(cudaMemcpyAsync(dk, hk + off, nb, cudaMemcpyDefault, pp.s_in), "cudaMemcpyAsync(k)")) != FA_OK ||
            (rc = ck(cudaMemcpyAsync(dv, hv + off, nb, cudaMemcpyDefault, pp.s_in), "cudaMemcpyAsync(v)")) != FA_OK ||
            (rc = ck(cudaEventRecord(pp.ev_in[b], pp.s_in), "cudaEventRecord")) != FA_OK)
            return rc;
        // the kernel on this chunk's heads
        if ((rc = ck(cudaStreamWaitEvent(pp.s_comp, pp.ev_in[b], 0), "cudaStreamWaitEvent")) != FA_OK) return rc;
        if ((rc = launch(dq, dk, dv, dout, dl, hc, pp.s_comp)) != FA_OK) return rc;
        if ((rc = ck(cudaEventRecord(pp.ev_comp[b], pp.s_comp), "cudaEventRecord")) != FA_OK) return rc;
        // copy-out
        if ((rc = ck(cudaStreamWaitEvent(pp.s_out, pp.ev_comp[b], 0), "cudaStreamWaitEvent")) != FA_OK ||
            (rc = ck(cudaMemcpyAsync(ho + ooff, dout, onb, cudaMemcpyDefault, pp.s_out), "cudaMemcpyAsync(o)")) != FA_OK ||
            (rc = ck(cudaMemcpyAsync(hl + loff, dl, lnb, cudaMemcpyDefault, pp.s_out), "cudaMemcpyAsync(lse)")) != FA_OK ||
            (rc = ck(cudaEventRecord(pp.ev_free[b], pp.s_out), "cudaEventRecord")) != FA_OK)
            return rc;
    }
    // the caller's stream continues once the last copy-out is done
    if ((rc = ck(cudaEventRecord(pp.ev_done, pp.s_out), "cudaEventRecord")) != FA_OK) return rc;
    return ck(cudaStreamWaitEvent(caller, pp.ev_done, 0), "cudaStreamWaitEvent");
}

}  // namespace

extern "C" int fa_fwd_host(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t H,
                           int64_t N, int64_t d, float scale, int causal, int dtype, void* stream) {
    g_last_error.clear();
    Sizes z;
    int rc = check_args(q, k, v, o, lse, B, H, N, d, scale, dtype, false, &z);
    if (rc != FA_OK) return rc;
    DeviceState* st = nullptr;
    if ((rc = device_state(&st)) != FA_OK) return rc;
    const size_t head_bytes = static_cast<size_t>(N * d * z.elem);
    return host_pipeline(q, k, v, o, lse, z.bh, N, head_bytes, head_bytes, static_cast<cudaStream_t>(stream),
                         [&](const void* dq, const void* dk, const void* dv, void* dout, float* dl, int64_t hc,
                             cudaStream_t s) {
                             return dispatch(st, dq, dk, dv, dout, dl, hc, N, d, scale, causal != 0, dtype, s);
                         });
}

// ---------------------------------------------------------------------------
// fa_decode: a few new queries over a key/value cache (split-KV, see
// fa_decode.cuh).  The chunking depends only on the arguments, so the
// workspace size can be computed before the call.
namespace {

constexpr int64_t kDecodeTargetCtas = 1184;  // 148 SMs x 8: the grid covers a B200 several times
constexpr int64_t kDecodeMinChunk = 256;     // keys; below this a CTA's fixed costs dominate

struct DecodePlan {
    int64_t bh = 0, groups = 0, chunks = 0, chunk = 0, nq_tile = 0;
    size_t part_bytes = 0, count_bytes = 0, workspace = 0;
};

// Queries per CTA: bf16 in groups of 16 on the warp MMA (one query too: the
// padded tile's tensor work is still far below the loads, and the swizzled
// tensor copies stream faster); fp32 on CUDA cores, one query or groups of 4.
int64_t decode_tile(int64_t nq, int dtype) {
    if (dtype == FA_DTYPE_BF16) return fa::decm::kQ;
    return nq == 1 ? 1 : fa::dec::kMaxQ;
}

DecodePlan decode_plan(int64_t bh, int64_t nq, int64_t nk, int64_t d, int64_t nq_tile) {
    DecodePlan pl;
    pl.bh = bh;
    pl.nq_tile = nq_tile;
    pl.groups = (nq + pl.nq_tile - 1) / pl.nq_tile;
    const int64_t ctas = bh * pl.groups;
    int64_t chunks = (kDecodeTargetCtas + ctas - 1) / ctas;
    const int64_t max_chunks = (nk + kDecodeMinChunk - 1) / kDecodeMinChunk;
    if (chunks > max_chunks) chunks = max_chunks;
    if (chunks < 1) chunks = 1;
    int64_t chunk = (nk + chunks - 1) / chunks;
    chunk = (chunk + fa::dec::kTileKeys - 1) / fa::dec::kTileKeys * fa::dec::kTileKeys;
    pl.chunk = chunk;
    pl.chunks = (nk + chunk - 1) / chunk;
    if (pl.chunks > 1) {
        pl.part_bytes = round_up(static_cast<size_t>(bh * nq * pl.chunks * (d + 2)) * 4, 256);
        pl.count_bytes = round_up(static_cast<size_t>(bh * pl.groups) * 4, 256);
    }
    pl.workspace = pl.part_bytes + pl.count_bytes;
    return pl;
}

int decode_check(const void* q, const void* k, const void* v, const void* o, const float* lse, int64_t B,
                 int64_t H, int64_t Nq, int64_t Nk, int64_t d, float scale, int causal, int dtype, DecodePlan* pl) {
    if (!q || !k || !v || !o || !lse) return fail(FA_ERR_INVALID_ARGUMENT, "null pointer argument");
    if (B < 1 || H < 1 || Nq < 1 || Nk < 1 || d < 1)
        return fail(FA_ERR_INVALID_ARGUMENT, "B, H, Nq, Nk and d must be >= 1");
    if (dtype != FA_DTYPE_F32 && dtype != FA_DTYPE_BF16) return fail(FA_ERR_INVALID_ARGUMENT, "unknown dtype");
    if (!std::isfinite(scale)) return fail(FA_ERR_INVALID_ARGUMENT, "scale must be finite");
    if (causal && Nq > Nk) return fail(FA_ERR_INVALID_ARGUMENT, "causal needs Nq <= Nk (the queries are the last Nq positions)");
    if (d != 64 && d != 128) return fail(FA_ERR_UNSUPPORTED, "head dim must be 64 or 128");
    if (Nk > (int64_t{1} << 30) || Nq > (int64_t{1} << 20)) return fail(FA_ERR_INVALID_ARGUMENT, "Nk or Nq too large");
    if (B > (int64_t{1} << 24) / H) return fail(FA_ERR_INVALID_ARGUMENT, "B * H too large");
    const int64_t bh = B * H;
    const int64_t elem = dtype == FA_DTYPE_BF16 ? 2 : 4;
    *pl = decode_plan(bh, Nq, Nk, d, decode_tile(Nq, dtype));
    if (pl->groups > 65535) return fail(FA_ERR_INVALID_ARGUMENT, "too many query groups");
    if (bh * pl->chunks > INT_MAX) return fail(FA_ERR_INVALID_ARGUMENT, "B * H * chunks too large");
    auto misaligned = [](const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) != 0; };
    if (misaligned(q, 16) || misaligned(k, 16) || misaligned(v, 16) || misaligned(o, 16))
        return fail(FA_ERR_INVALID_ARGUMENT, "q, k, v and o must be 16-byte aligned");
    if (misaligned(lse, 4)) return fail(FA_ERR_INVALID_ARGUMENT, "lse must be 4-byte aligned");
    const size_t qb = static_cast<size_t>(bh * Nq * d * elem), kb = static_cast<size_t>(bh * Nk * d * elem);
    const size_t lb = static_cast<size_t>(bh * Nq * 4);
    if (overlaps(o, qb, q, qb) || overlaps(o, qb, k, kb) || overlaps(o, qb, v, kb) || overlaps(o, qb, lse, lb))
        return fail(FA_ERR_INVALID_ARGUMENT, "o overlaps another argument");
    if (overlaps(lse, lb, q, qb) || overlaps(lse, lb, k, kb) || overlaps(lse, lb, v, kb))
        return fail(FA_ERR_INVALID_ARGUMENT, "lse overlaps another argument");
    return FA_OK;
}

template <typename T, int D, int NQ>
int launch_decode(DeviceState* st, int slot, const fa::dec::Params& p, const DecodePlan& pl, cudaStream_t s) {
    using C = fa::dec::Cfg<T, D>;
    auto kernel = fa::dec::fa_decode_kernel<T, D, NQ>;
    if (!st->decode_smem_raised[slot]) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(max dynamic shared memory)");
        std::lock_guard<std::mutex> lock(g_mu);
        st->decode_smem_raised[slot] = true;
    }
    dim3 grid(static_cast<unsigned>(pl.bh * pl.chunks), static_cast<unsigned>(pl.groups));
    kernel<<<grid, fa::dec::kThreads, C::kSmemBytes, s>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "launch of the decode kernel");
    return FA_OK;
}

template <int D>
int launch_decode_mma(DeviceState* st, int slot, const fa::dec::Params& p, const DecodePlan& pl, cudaStream_t s) {
    using C = fa::decm::Cfg<D>;
    auto kernel = fa::decm::fa_decode_mma_kernel<D>;
    if (!st->decode_mma_smem_raised[slot]) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(max dynamic shared memory)");
        std::lock_guard<std::mutex> lock(g_mu);
        st->decode_mma_smem_raised[slot] = true;
    }
    CUtensorMap tk, tv;
    int rc;
    if ((rc = encode_tile_map(&tk, p.k, pl.bh, p.nk, D, fa::dec::kTileKeys)) != FA_OK ||
        (rc = encode_tile_map(&tv, p.v, pl.bh, p.nk, D, fa::dec::kTileKeys)) != FA_OK)
        return rc;
    dim3 grid(static_cast<unsigned>(pl.bh * pl.chunks), static_cast<unsigned>(pl.groups));
    kernel<<<grid, fa::dec::kThreads, C::kSmemBytes, s>>>(tk, tv, p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "launch of the decode (warp MMA) kernel");
    return FA_OK;
}

}  // namespace

// The size covers either dtype's plan (the argument list has no dtype).
extern "C" size_t fa_decode_workspace_bytes(int64_t B, int64_t H, int64_t Nq, int64_t Nk, int64_t d) {
    if (B < 1 || H < 1 || Nq < 1 || Nk < 1 || d < 1 || B > (int64_t{1} << 24) / H) return 0;
    const size_t a = decode_plan(B * H, Nq, Nk, d, decode_tile(Nq, FA_DTYPE_BF16)).workspace;
    const size_t b = decode_plan(B * H, Nq, Nk, d, decode_tile(Nq, FA_DTYPE_F32)).workspace;
    return a > b ? a : b;
}

extern "C" int fa_decode(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t H,
                         int64_t Nq, int64_t Nk, int64_t d, float scale, int causal, int dtype, void* workspace,
                         size_t workspace_bytes, void* stream) {
    g_last_error.clear();
    DecodePlan pl;
    int rc = decode_check(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, dtype, &pl);
    if (rc != FA_OK) return rc;
    if (pl.workspace > 0) {
        if (!workspace || workspace_bytes < pl.workspace)
            return fail(FA_ERR_INVALID_ARGUMENT, "workspace missing or smaller than fa_decode_workspace_bytes()");
        if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0)
            return fail(FA_ERR_INVALID_ARGUMENT, "workspace must be 256-byte aligned");
    }
    DeviceState* st = nullptr;
    if ((rc = device_state(&st)) != FA_OK) return rc;
    fa::dec::Params p;
    p.q = q;
    p.k = k;
    p.v = v;
    p.o = o;
    p.lse = lse;
    p.part = pl.workspace ? static_cast<float*>(workspace) : nullptr;
    p.count = pl.workspace ? reinterpret_cast<unsigned*>(static_cast<char*>(workspace) + pl.part_bytes) : nullptr;
    p.status = st->status;
    p.nq = static_cast<int>(Nq);
    p.nk = static_cast<int>(Nk);
    p.chunk = static_cast<int>(pl.chunk);
    p.chunks = static_cast<int>(pl.chunks);
    p.groups = static_cast<int>(pl.groups);
    p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    p.causal = causal != 0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the chunk counters start from zero on every call (the workspace may
    // have held other sizes' partials since)
    if (pl.workspace > 0) {
        cudaError_t e = cudaMemsetAsync(p.count, 0, pl.count_bytes, s);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(decode counters)");
    }
    const bool one = pl.nq_tile == 1;
    if (dtype == FA_DTYPE_BF16)
        return d == 128 ? launch_decode_mma<128>(st, 0, p, pl, s) : launch_decode_mma<64>(st, 1, p, pl, s);
    if (d == 128) return one ? launch_decode<float, 128, 1>(st, 4, p, pl, s)
                             : launch_decode<float, 128, fa::dec::kMaxQ>(st, 5, p, pl, s);
    return one ? launch_decode<float, 64, 1>(st, 6, p, pl, s) : launch_decode<float, 64, fa::dec::kMaxQ>(st, 7, p, pl, s);
}

// ---------------------------------------------------------------------------
// fa_bwd: gradients (see fa_bwd_tc.cuh).  Workspace, every array padded to
// whole 128-row blocks per head (npad rows): L = -lse * log2(e) and
// D = rowsum(dO * O), [B*H][npad] fp32 each, then the fp32 dQ accumulator
// [B*H][npad][d].
namespace {

struct BwdWorkspace {
    size_t vec_bytes = 0;  // one of the two row vectors, rounded up to 256
    size_t total = 0;
};

BwdWorkspace bwd_workspace_layout(int64_t bh, int64_t npad, int64_t d) {
    BwdWorkspace w;
    w.vec_bytes = round_up(static_cast<size_t>(bh * npad) * 4, 256);
    w.total = 2 * w.vec_bytes + round_up(static_cast<size_t>(bh * npad * d) * 4, 256);
    return w;
}

// 3-D view (d, npad, B*H) of the fp32 dQ accumulator, boxes of 32 columns x
// 32 rows with 128-byte swizzle: the unit of the kernel's reduce-adds.
int encode_dq_acc_map(CUtensorMap* map, float* ptr, int64_t bh, int64_t npad, int64_t d) {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(npad), static_cast<cuuint64_t>(bh)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d * 4), static_cast<cuuint64_t>(npad * d * 4)};
    cuuint32_t box[3] = {32, 32, 1};
    cuuint32_t elem[3] = {1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, ptr, dims, strides, box, elem,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled (dQ accumulator) failed with CUresult " + std::to_string(r));
    return FA_OK;
}

template <int D, bool kCausal>
int launch_bwd(DeviceState* st, int slot, const void* q, const void* k, const void* v, const void* o,
               const float* lse, const void* dout, void* dq, void* dk, void* dv, void* workspace, int64_t bh,
               int64_t n, float scale, cudaStream_t s) {
    using L = fa::bwd::Layout<D>;
    auto kernel = fa::bwd::fa_bwd_kernel<D, kCausal>;
    cudaError_t e;
    if (!st->bwd_smem_raised[slot]) {
        if ((e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmemBytes)) != cudaSuccess)
            return cuda_fail(e, "cudaFuncSetAttribute(max dynamic shared memory)");
        std::lock_guard<std::mutex> lock(g_mu);
        st->bwd_smem_raised[slot] = true;
    }
    const int64_t nblocks = (n + fa::bwd::kBlock - 1) / fa::bwd::kBlock;
    const int64_t npad = nblocks * fa::bwd::kBlock;
    const BwdWorkspace ws = bwd_workspace_layout(bh, npad, D);
    float* lvec = static_cast<float*>(workspace);
    float* dvec = reinterpret_cast<float*>(static_cast<char*>(workspace) + ws.vec_bytes);
    float* dq_acc = reinterpret_cast<float*>(static_cast<char*>(workspace) + 2 * ws.vec_bytes);
    const int64_t prows = bh * npad;
    constexpr int64_t kPrepRows = 256 / (D / 8);  // rows per 256-thread block
    fa::bwd::fa_bwd_prep_kernel<D><<<static_cast<unsigned>((prows + kPrepRows - 1) / kPrepRows), 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(dout), static_cast<const __nv_bfloat16*>(o), lse, lvec, dvec, dq_acc, bh,
        static_cast<int>(n), static_cast<int>(npad));
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "launch of the backward preparation kernel");
    CUtensorMap tq, tk, tv, tdo, tdq;
    int rc;
    if ((rc = encode_tile_map(&tq, q, bh, n, D)) != FA_OK || (rc = encode_tile_map(&tk, k, bh, n, D)) != FA_OK ||
        (rc = encode_tile_map(&tv, v, bh, n, D)) != FA_OK || (rc = encode_tile_map(&tdo, dout, bh, n, D)) != FA_OK ||
        (rc = encode_dq_acc_map(&tdq, dq_acc, bh, npad, D)) != FA_OK)
        return rc;
    fa::bwd::Params p;
    p.dk = static_cast<__nv_bfloat16*>(dk);
    p.dv = static_cast<__nv_bfloat16*>(dv);
    p.lvec = lvec;
    p.dvec = dvec;
    p.status = st->status;
    p.n = static_cast<int>(n);
    p.npad = static_cast<int>(npad);
    p.nblocks = static_cast<int>(nblocks);
    p.bh = static_cast<int>(bh);
    p.scale = scale;
    p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    kernel<<<static_cast<unsigned>(nblocks * bh), fa::bwd::kThreads, L::kSmemBytes, s>>>(tq, tk, tv, tdo, tdq, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "launch of the backward kernel");
    const int64_t vecs = bh * n * (D / 8);
    const int64_t cap = static_cast<int64_t>(st->sm_count) * 8;
    const unsigned blocks = static_cast<unsigned>(std::min<int64_t>((vecs + 255) / 256, cap));
    fa::bwd::fa_bwd_dq_convert_kernel<D><<<blocks, 256, 0, s>>>(dq_acc, static_cast<__nv_bfloat16*>(dq), bh,
                                                                static_cast<int>(n), static_cast<int>(npad), scale);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "launch of the dQ conversion kernel");
    return FA_OK;
}

}  // namespace

extern "C" size_t fa_bwd_workspace_bytes(int64_t B, int64_t H, int64_t N, int64_t d) {
    if (B < 1 || H < 1 || N < 1 || (d != 64 && d != 128) || B > (int64_t{1} << 24) / H || N > (int64_t{1} << 30))
        return 0;
    const int64_t npad = (N + fa::bwd::kBlock - 1) / fa::bwd::kBlock * fa::bwd::kBlock;
    return bwd_workspace_layout(B * H, npad, d).total;
}

extern "C" int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                      void* dq, void* dk, void* dv, int64_t B, int64_t H, int64_t N, int64_t d, float scale,
                      int causal, int dtype, void* workspace, size_t workspace_bytes, void* stream) {
    g_last_error.clear();
    if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv)
        return fail(FA_ERR_INVALID_ARGUMENT, "null pointer argument");
    if (B < 1 || H < 1 || N < 1 || d < 1) return fail(FA_ERR_INVALID_ARGUMENT, "B, H, N and d must be >= 1");
    if (dtype != FA_DTYPE_F32 && dtype != FA_DTYPE_BF16) return fail(FA_ERR_INVALID_ARGUMENT, "unknown dtype");
    if (!std::isfinite(scale)) return fail(FA_ERR_INVALID_ARGUMENT, "scale must be finite");
    if (dtype != FA_DTYPE_BF16) return fail(FA_ERR_UNSUPPORTED, "the backward pass takes bf16 tensors");
    if (d != 64 && d != 128) return fail(FA_ERR_UNSUPPORTED, "head dim must be 64 or 128");
    if (N > (int64_t{1} << 30) || B > 65535 / H) return fail(FA_ERR_INVALID_ARGUMENT, "B * H or N too large");
    if ((N + fa::bwd::kBlock - 1) / fa::bwd::kBlock * B * H > INT_MAX)
        return fail(FA_ERR_INVALID_ARGUMENT, "B * H * N too large");
    const int64_t bh = B * H;
    const size_t tb = static_cast<size_t>(bh * N * d * 2), lb = static_cast<size_t>(bh * N * 4);
    const size_t need = fa_bwd_workspace_bytes(B, H, N, d);
    if (!workspace || workspace_bytes < need) return fail(FA_ERR_INVALID_ARGUMENT, "workspace missing or too small");
    auto mis = [](const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) != 0; };
    if (mis(q, 16) || mis(k, 16) || mis(v, 16) || mis(o, 16) || mis(dout, 16) || mis(dq, 16) || mis(dk, 16) ||
        mis(dv, 16) || mis(workspace, 16))
        return fail(FA_ERR_INVALID_ARGUMENT, "tensors and workspace must be 16-byte aligned");
    if (mis(lse, 4)) return fail(FA_ERR_INVALID_ARGUMENT, "lse must be 4-byte aligned");
    const void* ins[6] = {q, k, v, o, dout, lse};
    const size_t insz[6] = {tb, tb, tb, tb, tb, lb};
    void* outs[4] = {dq, dk, dv, workspace};
    const size_t outsz[4] = {tb, tb, tb, need};
    for (int a = 0; a < 4; ++a) {
        for (int b = 0; b < 6; ++b)
            if (overlaps(outs[a], outsz[a], ins[b], insz[b]))
                return fail(FA_ERR_INVALID_ARGUMENT, "an output or the workspace overlaps an input");
        for (int b = a + 1; b < 4; ++b)
            if (overlaps(outs[a], outsz[a], outs[b], outsz[b]))
                return fail(FA_ERR_INVALID_ARGUMENT, "outputs overlap each other");
    }
    DeviceState* st = nullptr;
    int rc = device_state(&st);
    if (rc != FA_OK) return rc;
    if (st->cc_major != 10) return fail(FA_ERR_UNSUPPORTED, "the backward kernels need an sm_100 (B200-class) GPU");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool c = causal != 0;
    if (d == 128) return c ? launch_bwd<128, true>(st, 0, q, k, v, o, lse, dout, dq, dk, dv, workspace, bh, N, scale, s)
                           : launch_bwd<128, false>(st, 1, q, k, v, o, lse, dout, dq, dk, dv, workspace, bh, N, scale, s);
    return c ? launch_bwd<64, true>(st, 2, q, k, v, o, lse, dout, dq, dk, dv, workspace, bh, N, scale, s)
             : launch_bwd<64, false>(st, 3, q, k, v, o, lse, dout, dq, dk, dv, workspace, bh, N, scale, s);
}

// ---------------------------------------------------------------------------
// fa_merge: attention results over disjoint key sets -> the result over their
// union (see fa_merge.cuh).
extern "C" int fa_merge(const void* o_parts, const float* lse_parts, int64_t parts, int64_t rows, int64_t d,
                        void* o, float* lse, int dtype, void* stream) {
    g_last_error.clear();
    if (!o_parts || !lse_parts || !o || !lse) return fail(FA_ERR_INVALID_ARGUMENT, "null pointer argument");
    if (parts < 1 || rows < 1 || d < 1) return fail(FA_ERR_INVALID_ARGUMENT, "parts, rows and d must be >= 1");
    if (dtype != FA_DTYPE_F32 && dtype != FA_DTYPE_BF16) return fail(FA_ERR_INVALID_ARGUMENT, "unknown dtype");
    if (d != 64 && d != 128) return fail(FA_ERR_UNSUPPORTED, "head dim must be 64 or 128");
    if (parts > 65536 || rows > (int64_t{1} << 40) / parts) return fail(FA_ERR_INVALID_ARGUMENT, "sizes too large");
    const int64_t elem = dtype == FA_DTYPE_BF16 ? 2 : 4;
    auto mis = [](const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) != 0; };
    if (mis(o_parts, 16) || mis(o, 16)) return fail(FA_ERR_INVALID_ARGUMENT, "o_parts and o must be 16-byte aligned");
    if (mis(lse_parts, 4) || mis(lse, 4)) return fail(FA_ERR_INVALID_ARGUMENT, "lse arrays must be 4-byte aligned");
    const size_t ob = static_cast<size_t>(rows * d * elem), lb = static_cast<size_t>(rows * 4);
    if (overlaps(o, ob, o_parts, ob * parts) || overlaps(o, ob, lse_parts, lb * parts) || overlaps(o, ob, lse, lb) ||
        overlaps(lse, lb, o_parts, ob * parts) || overlaps(lse, lb, lse_parts, lb * parts))
        return fail(FA_ERR_INVALID_ARGUMENT, "outputs overlap the inputs");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const unsigned blocks = static_cast<unsigned>((rows + 7) / 8);
    const int np = static_cast<int>(parts);
    if (dtype == FA_DTYPE_BF16) {
        if (d == 128)
            fa::merge::fa_merge_kernel<__nv_bfloat16, 128><<<blocks, 256, 0, s>>>(
                static_cast<const __nv_bfloat16*>(o_parts), lse_parts, np, rows, static_cast<__nv_bfloat16*>(o), lse);
        else
            fa::merge::fa_merge_kernel<__nv_bfloat16, 64><<<blocks, 256, 0, s>>>(
                static_cast<const __nv_bfloat16*>(o_parts), lse_parts, np, rows, static_cast<__nv_bfloat16*>(o), lse);
    } else {
        if (d == 128)
            fa::merge::fa_merge_kernel<float, 128><<<blocks, 256, 0, s>>>(
                static_cast<const float*>(o_parts), lse_parts, np, rows, static_cast<float*>(o), lse);
        else
            fa::merge::fa_merge_kernel<float, 64><<<blocks, 256, 0, s>>>(
                static_cast<const float*>(o_parts), lse_parts, np, rows, static_cast<float*>(o), lse);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "launch of the merge kernel");
    return FA_OK;
}

// ---------------------------------------------------------------------------
// fa_fwd_fp8: the forward with E4M3 inputs (see fa_fwd_fp8_tc.cuh).
namespace {

// 3-D view (d, N, B*H) of a [B*H][N][128] one-byte tensor, boxes of
// 128 x 128 x 1 (one 128-byte swizzle panel); rows past N read as zeros.
int encode_tile_map_u8(CUtensorMap* map, const void* ptr, int64_t bh, int64_t n) {
    cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(n), static_cast<cuuint64_t>(bh)};
    cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(n * 128)};
    cuuint32_t box[3] = {128, static_cast<cuuint32_t>(fa::tc::kBlockM), 1};
    cuuint32_t elem[3] = {1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box, elem,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled failed with CUresult " + std::to_string(r));
    return FA_OK;
}

template <bool kCausal>
int launch_e4m3(DeviceState* st, const void* q, const void* k, const void* v, void* o, float* lse, int64_t bh,
                int64_t n, double scale_qk, float o_scale, cudaStream_t stream) {
    using L = fa::tc8::Layout;
    auto kernel = fa::tc8::fa_fwd_e4m3_kernel<kCausal>;
    if (!st->fp8_smem_raised[kCausal ? 0 : 1]) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmemBytes);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(max dynamic shared memory)");
        std::lock_guard<std::mutex> lock(g_mu);
        st->fp8_smem_raised[kCausal ? 0 : 1] = true;
    }
    CUtensorMap tq, tk, tv;
    int rc;
    if ((rc = encode_tile_map_u8(&tq, q, bh, n)) != FA_OK) return rc;
    if ((rc = encode_tile_map_u8(&tk, k, bh, n)) != FA_OK) return rc;
    if ((rc = encode_tile_map_u8(&tv, v, bh, n)) != FA_OK) return rc;

    fa::tc8::Params p;
    p.base.o = static_cast<__nv_bfloat16*>(o);
    p.base.lse = lse;
    p.base.status = st->status;
    p.base.sched = st->queues + 2 * (st->next_queue.fetch_add(1, std::memory_order_relaxed) % kQueues);
    p.base.bh = static_cast<int>(bh);
    p.base.n = static_cast<int>(n);
    p.base.num_qblocks = static_cast<int>((n + fa::tc::kUnitRows - 1) / fa::tc::kUnitRows);
    p.base.num_kblocks = static_cast<int>((n + fa::tc::kBlockN - 1) / fa::tc::kBlockN);
    p.base.num_units = p.base.bh * p.base.num_qblocks;
    p.base.scale_log2 = static_cast<float>(scale_qk * 1.4426950408889634);
    p.base.skip_one_arrival = 0;
    p.base.clock = st->clock;
    p.o_scale = o_scale;
    const int grid = p.base.num_units < st->sm_count ? p.base.num_units : st->sm_count;
    cudaError_t e = launch_overlapped(kernel, grid, fa::tc8::kThreads, L::kSmemBytes, stream, tq, tk, tv, p);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "launch of the E4M3 attention kernel");
    return FA_OK;
}

}  // namespace

namespace {

// Arguments of the E4M3 forward; device_pointers adds the alignment checks.
int check_fp8_args(const void* q, const void* k, const void* v, const void* o, const float* lse, int64_t B,
                   int64_t H, int64_t N, int64_t d, float scale, float descale_q, float descale_k, float descale_v,
                   bool device_pointers, int64_t* bh_out, double* scale_qk_out) {
    if (!q || !k || !v || !o || !lse) return fail(FA_ERR_INVALID_ARGUMENT, "null pointer argument");
    if (B < 1 || H < 1 || N < 1 || d < 1) return fail(FA_ERR_INVALID_ARGUMENT, "B, H, N and d must be >= 1");
    if (!std::isfinite(scale) || !std::isfinite(descale_q) || !std::isfinite(descale_k) || !std::isfinite(descale_v))
        return fail(FA_ERR_INVALID_ARGUMENT, "scale and descale factors must be finite");
    const double scale_qk = static_cast<double>(scale) * descale_q * descale_k;
    if (!std::isfinite(static_cast<float>(scale_qk * 1.4426950408889634)))
        return fail(FA_ERR_INVALID_ARGUMENT, "scale * descale_q * descale_k overflows fp32");
    if (d != 128) return fail(FA_ERR_UNSUPPORTED, "the E4M3 forward takes head dim 128");
    if (B > INT_MAX / H) return fail(FA_ERR_INVALID_ARGUMENT, "B * H too large");
    const int64_t bh = B * H;
    if (N > (int64_t{1} << 30)) return fail(FA_ERR_INVALID_ARGUMENT, "N too large (max 2^30)");
    if (bh * ((N + 255) / 256) > INT_MAX) return fail(FA_ERR_INVALID_ARGUMENT, "B * H * N too large");
    if (bh > (int64_t{1} << 62) / (N * d * 2)) return fail(FA_ERR_INVALID_ARGUMENT, "tensor size overflows");
    const size_t in_bytes = static_cast<size_t>(bh * N * d), o_bytes = 2 * in_bytes;
    const size_t lse_bytes = static_cast<size_t>(bh * N * 4);
    auto mis = [](const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) != 0; };
    if (device_pointers) {
        if (mis(q, 16) || mis(k, 16) || mis(v, 16) || mis(o, 16))
            return fail(FA_ERR_INVALID_ARGUMENT, "q, k, v and o must be 16-byte aligned");
        if (mis(lse, 4)) return fail(FA_ERR_INVALID_ARGUMENT, "lse must be 4-byte aligned");
    }
    if (overlaps(o, o_bytes, q, in_bytes) || overlaps(o, o_bytes, k, in_bytes) || overlaps(o, o_bytes, v, in_bytes) ||
        overlaps(o, o_bytes, lse, lse_bytes))
        return fail(FA_ERR_INVALID_ARGUMENT, "o overlaps another argument");
    if (overlaps(lse, lse_bytes, q, in_bytes) || overlaps(lse, lse_bytes, k, in_bytes) ||
        overlaps(lse, lse_bytes, v, in_bytes))
        return fail(FA_ERR_INVALID_ARGUMENT, "lse overlaps another argument");
    *bh_out = bh;
    *scale_qk_out = scale_qk;
    return FA_OK;
}

int e4m3_launch(DeviceState* st, const void* q, const void* k, const void* v, void* o, float* lse, int64_t bh,
                int64_t N, double scale_qk, float descale_v, bool causal, cudaStream_t s) {
    return causal ? launch_e4m3<true>(st, q, k, v, o, lse, bh, N, scale_qk, descale_v, s)
                  : launch_e4m3<false>(st, q, k, v, o, lse, bh, N, scale_qk, descale_v, s);
}

}  // namespace

extern "C" int fa_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t H,
                          int64_t N, int64_t d, float scale, float descale_q, float descale_k, float descale_v,
                          int causal, void* stream) {
    g_last_error.clear();
    int64_t bh = 0;
    double scale_qk = 0.0;
    int rc = check_fp8_args(q, k, v, o, lse, B, H, N, d, scale, descale_q, descale_k, descale_v, true, &bh,
                            &scale_qk);
    if (rc != FA_OK) return rc;
    DeviceState* st = nullptr;
    if ((rc = device_state(&st)) != FA_OK) return rc;
    if (st->cc_major != 10) return fail(FA_ERR_UNSUPPORTED, "the E4M3 kernel needs an sm_100 (B200-class) GPU");
    return e4m3_launch(st, q, k, v, o, lse, bh, N, scale_qk, descale_v, causal != 0, static_cast<cudaStream_t>(stream));
}

extern "C" int fa_fwd_fp8_host(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B,
                               int64_t H, int64_t N, int64_t d, float scale, float descale_q, float descale_k,
                               float descale_v, int causal, void* stream) {
    g_last_error.clear();
    int64_t bh = 0;
    double scale_qk = 0.0;
    int rc = check_fp8_args(q, k, v, o, lse, B, H, N, d, scale, descale_q, descale_k, descale_v, false, &bh,
                            &scale_qk);
    if (rc != FA_OK) return rc;
    DeviceState* st = nullptr;
    if ((rc = device_state(&st)) != FA_OK) return rc;
    if (st->cc_major != 10) return fail(FA_ERR_UNSUPPORTED, "the E4M3 kernel needs an sm_100 (B200-class) GPU");
    const size_t head_in = static_cast<size_t>(N * d);  // one byte per element in, bf16 out
    return host_pipeline(q, k, v, o, lse, bh, N, head_in, 2 * head_in, static_cast<cudaStream_t>(stream),
                         [&](const void* dq, const void* dk, const void* dv, void* dout, float* dl, int64_t hc,
                             cudaStream_t s) {
                             return e4m3_launch(st, dq, dk, dv, dout, dl, hc, N, scale_qk, descale_v, causal != 0, s);
                         });
}
