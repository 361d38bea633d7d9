// read_rate.cu -- jano_stream_sum: one streaming pass over a float buffer,
// the ceiling that the analyzer's HBM rate is measured against.
//
// The analyzer reads its latent history once.  How fast one pass over a
// buffer of that size can go at all on this device -- with the launch, the
// ramp-up of the memory pipeline and the tail included -- is what its
// fraction of the HBM copy rate should be compared with.  This kernel does
// nothing but that pass with the least work per byte: a persistent grid
// (one CTA per SM by default), each CTA streaming its contiguous share of the
// buffer through a deep shared-memory ring filled by 1-D bulk copies
// (cp.async.bulk, no tensor map), the consumer warps adding the floats
// (fixed order, so the result is deterministic) and writing one partial sum
// per CTA.  Every wait is bounded.
#include "jano_common.cuh"

namespace jano {
namespace {

constexpr int kConsumerWarps = 8;
constexpr int kThreads = (kConsumerWarps + 1) * 32;     // + one producer warp
constexpr int kStageBytes = 16 * 1024;
constexpr int kStages = 12;                              // 192 KB of ring per CTA
constexpr long long kWaitLimit = 1ll << 31;

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}

// Bounded wait that gives up as soon as another thread of the CTA recorded a
// timeout (abort flag in shared memory).
__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, int* err,
                                              volatile int* abort) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    for (;;) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
        if (clock64() - t0 > kWaitLimit) {
            *abort = 1;
            raise_error(err, JANO_ETIMEOUT);
            return false;
        }
    }
}

__global__ void __launch_bounds__(kThreads, 1)
stream_sum_kernel(const float4* __restrict__ x, long long n4, float* __restrict__ partial, int* err) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = ptx::smem_u32(smem_raw);
    const uint32_t base = (raw + 127u) & ~127u;
    uint8_t* gbase = smem_raw + (base - raw);
    const uint32_t bars = base + kStages * kStageBytes;       // kStages full, kStages empty
    volatile int* abort = reinterpret_cast<volatile int*>(gbase + kStages * kStageBytes + 16 * kStages);
    __shared__ float wsum[kConsumerWarps];
    auto full = [&](int s) { return bars + 8u * s; };
    auto empty = [&](int s) { return bars + 8u * (kStages + s); };

    // this CTA's share, in whole float4s
    const long long per = (n4 + gridDim.x - 1) / gridDim.x;
    const long long lo = min(n4, (long long)blockIdx.x * per), hi = min(n4, lo + per);
    const long long bytes = (hi - lo) * 16;
    const int n_stages = (int)((bytes + kStageBytes - 1) / kStageBytes);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(full(s), 1);
            ptx::mbar_init(empty(s), kConsumerWarps);
        }
        *abort = 0;
        ptx::fence_mbar_init();
    }
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp == kConsumerWarps) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const char* src = reinterpret_cast<const char*>(x + lo);
            int last[kStages];
            for (int s = 0; s < kStages; ++s) last[s] = -1;
            for (int i = 0; i < n_stages; ++i) {
                const int s = i % kStages;
                if (!wait_or_abort(empty(s), ((i / kStages) & 1) ^ 1, err, abort)) break;
                const long long off = (long long)i * kStageBytes;
                const uint32_t nb = (uint32_t)min((long long)kStageBytes, bytes - off);
                ptx::mbar_arrive_expect_tx(full(s), nb);
                bulk_load(base + s * kStageBytes, src + off, nb, full(s));
                last[s] = i;
            }
            // drain: every copy issued lands before the CTA's shared memory is released
            for (int s = 0; s < kStages; ++s)
                if (last[s] >= 0) ptx::mbar_wait(full(s), (last[s] / kStages) & 1, kWaitLimit);
        }
        return;
    }
    // ---------------------------------------------------------------- consumers
    float acc = 0.f;
    for (int i = 0; i < n_stages; ++i) {
        const int s = i % kStages;
        if (!wait_or_abort(full(s), (i / kStages) & 1, err, abort)) break;
        const long long off = (long long)i * kStageBytes;
        const int nv = (int)(min((long long)kStageBytes, bytes - off) / 16);
        const float4* st = reinterpret_cast<const float4*>(gbase + s * kStageBytes);
        for (int v = threadIdx.x; v < nv; v += kConsumerWarps * 32) {
            const float4 q = st[v];
            acc += (q.x + q.y) + (q.z + q.w);
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(empty(s));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
    if (lane == 0) wsum[warp] = acc;
    asm volatile("bar.sync 1, %0;" ::"r"(kConsumerWarps * 32) : "memory");
    if (threadIdx.x == 0) {
        float t = 0.f;
        for (int w = 0; w < kConsumerWarps; ++w) t += wsum[w];
        partial[blockIdx.x] = t;
    }
}

}  // namespace

cudaError_t launch_stream_sum(const float* x, long long n, float* partial, int n_partial, int* err,
                              cudaStream_t st) {
    static DeviceOnce opted_in;
    int dev = 0;
    cudaGetDevice(&dev);
    const int smem = kStages * kStageBytes + 16 * kStages + 16 + 128;
    if (!opted_in.done(dev)) {
        cudaError_t e = cudaFuncSetAttribute(stream_sum_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        opted_in.mark(dev);
    }
    stream_sum_kernel<<<n_partial, kThreads, smem, st>>>(reinterpret_cast<const float4*>(x), n / 4, partial,
                                                          err);
    return cudaGetLastError();
}

}  // namespace jano
