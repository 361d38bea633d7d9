// classify.cu -- three-level split of block scores (Jano pages: nl technical
// summary, Methodologie 1 "Resultaat": Level 1 Static, 2 Moderate, 3 Active;
// zh 2.2 item 1).
//
// Blocks are ranked by the key (score, block index).  A block is Static when
// its rank is below k_static = n_S and Active when its rank is at least
// k_active = n - n_A.  Instead of sorting, one thread block finds, for each
// of the two rank thresholds, the 32-bit score key sitting at that rank with
// an MSB-first radix select (4 passes of 8-bit digits, shared-memory
// histograms), then one pass in index order resolves ties at the threshold
// value with a block-wide ballot scan: among equal scores the lower block
// index ranks lower.  Exact and deterministic; no scratch memory.  The n
// scores are re-read from L2 on each pass (n is at most a few 10^5).
#include "jano_common.cuh"

namespace jano {
namespace {

constexpr int kThreads = 1024;
constexpr int kChunk = 8;    // independent loads in flight per thread

// Order-preserving map float -> uint32 (unsigned order == float order),
// with -0 folded onto +0.
__device__ __forceinline__ uint32_t order_key(uint32_t b) {
    if (b == 0x80000000u) b = 0u;
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__global__ void __launch_bounds__(kThreads, 1)
classify_kernel(const uint32_t* __restrict__ bits, int n, long long k_static,
                long long k_active, uint8_t* __restrict__ levels, int* err) {
    __shared__ unsigned hist[2][256];
    __shared__ unsigned s_val[2];
    __shared__ unsigned s_need[2];
    __shared__ unsigned s_wtot[2][32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // targets: t=0 -> rank k_static, t=1 -> rank k_active; "live" if 0 < k < n
    const long long ks[2] = {k_static, k_active};
    const bool live0 = k_static > 0 && k_static < n;
    const bool live1 = k_active > 0 && k_active < n;

    // ---- pass 0: reject non-finite scores -----------------------------------
    int bad = 0;
    for (int base = 0; base < n; base += kThreads * kChunk) {
        uint32_t v[kChunk];
#pragma unroll
        for (int j = 0; j < kChunk; ++j) {
            const int i = base + j * kThreads + tid;
            v[j] = i < n ? __ldg(bits + i) : 0u;
        }
#pragma unroll
        for (int j = 0; j < kChunk; ++j) bad |= (v[j] & 0x7F800000u) == 0x7F800000u;
    }
    if (__syncthreads_or(bad)) {
        if (tid == 0) raise_error(err, JANO_ENONFINITE);
        return;
    }

    if (tid < 2) {
        s_val[tid] = 0u;
        s_need[tid] = (unsigned)(ks[tid] < 0 ? 0 : (ks[tid] > n ? n : ks[tid]));
    }

    // ---- radix select, most significant digit first -------------------------
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        const uint32_t hi_mask = pass == 0 ? 0u : (0xFFFFFFFFu << (shift + 8));
        for (int b = tid; b < 512; b += kThreads) (&hist[0][0])[b] = 0u;
        __syncthreads();
        const uint32_t p0 = s_val[0] & hi_mask, p1 = s_val[1] & hi_mask;
        for (int base = 0; base < n; base += kThreads * kChunk) {
            uint32_t v[kChunk];
#pragma unroll
            for (int j = 0; j < kChunk; ++j) {
                const int i = base + j * kThreads + tid;
                v[j] = i < n ? order_key(__ldg(bits + i)) : 0u;
            }
#pragma unroll
            for (int j = 0; j < kChunk; ++j) {
                if (base + j * kThreads + tid < n) {
                    const uint32_t dg = (v[j] >> shift) & 0xFFu;
                    if (live0 && (v[j] & hi_mask) == p0) atomicAdd(&hist[0][dg], 1u);
                    if (live1 && (v[j] & hi_mask) == p1) atomicAdd(&hist[1][dg], 1u);
                }
            }
        }
        __syncthreads();
        if (warp < 2 && (warp == 0 ? live0 : live1)) {
            // lane owns bins [8*lane, 8*lane+8)
            unsigned c[8], s = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) { c[j] = hist[warp][8 * lane + j]; s += c[j]; }
            unsigned incl = s;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                if (lane >= o) incl += y;
            }
            const unsigned need = s_need[warp];
            const unsigned excl = incl - s;
            // the lane whose range holds the need-th candidate (0-based)
            const bool mine = excl <= need && need < incl;
            if (mine) {
                unsigned acc = excl;
                int dg = 8 * lane;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (acc + c[j] > need) { dg = 8 * lane + j; break; }
                    acc += c[j];
                }
                s_val[warp] |= (uint32_t)dg << shift;
                s_need[warp] = need - acc;
            }
        }
        __syncthreads();
    }

    // ---- final pass: ties at the threshold value resolved by block index ----
    const uint32_t v0 = s_val[0], v1 = s_val[1];
    const unsigned need0 = s_need[0], need1 = s_need[1];
    unsigned run0 = 0, run1 = 0;
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int base = 0; base < n; base += kThreads) {
        const int i = base + tid;
        const bool ok = i < n;
        const uint32_t u = ok ? order_key(__ldg(bits + i)) : 0u;
        const bool e0 = ok && live0 && u == v0;
        const bool e1 = ok && live1 && u == v1;
        const unsigned b0 = __ballot_sync(0xFFFFFFFFu, e0);
        const unsigned b1 = __ballot_sync(0xFFFFFFFFu, e1);
        if (lane == 0) { s_wtot[0][warp] = __popc(b0); s_wtot[1][warp] = __popc(b1); }
        __syncthreads();
        unsigned pre0 = 0, pre1 = 0, tot0 = 0, tot1 = 0;
        for (int w = 0; w < kThreads / 32; ++w) {
            const unsigned a0 = s_wtot[0][w], a1 = s_wtot[1][w];
            if (w < warp) { pre0 += a0; pre1 += a1; }
            tot0 += a0;
            tot1 += a1;
        }
        if (ok) {
            const unsigned tie0 = run0 + pre0 + __popc(b0 & lt_mask);
            const unsigned tie1 = run1 + pre1 + __popc(b1 & lt_mask);
            // rank < k_static ?
            const bool below_s = live0 ? (u < v0 || (e0 && tie0 < need0)) : (k_static >= n);
            // rank < k_active ?
            const bool below_a = live1 ? (u < v1 || (e1 && tie1 < need1)) : (k_active >= n);
            levels[i] = below_s ? 1 : (below_a ? 2 : 3);
        }
        run0 += tot0;
        run1 += tot1;
        __syncthreads();
    }
}

}  // namespace

cudaError_t launch_classify(const float* scores, int n, long long k_static,
                            long long k_active, uint8_t* levels, int* err,
                            cudaStream_t st) {
    classify_kernel<<<1, kThreads, 0, st>>>(reinterpret_cast<const uint32_t*>(scores), n,
                                            k_static, k_active, levels, err);
    return cudaGetLastError();
}

}  // namespace jano
