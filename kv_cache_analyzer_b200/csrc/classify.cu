// classify.cu -- three-level split of block scores (Jano pages: nl technical
// summary, Methodologie 1 "Resultaat": Level 1 Static, 2 Moderate, 3 Active;
// zh 2.2 item 1).
//
// Blocks are ranked by the key (score, block index).  A block is Static when
// its rank is below k_static = n_S and Active when its rank is at least
// k_active = n - n_A.  Instead of sorting, the kernel finds, for each of the
// two rank thresholds, the 32-bit order-preserving score key at that rank by
// a most-significant-first radix select, then resolves ties at the threshold
// value by block index in one pass in index order.
//
// The select works on the range of keys that occur, [min, max]: each pass
// splits the current bucket of both targets into 2048 bins of 2^shift keys
// (the first bucket is the whole range, so the bins spread over the keys
// present and shared-memory atomics rarely collide), keeps the bin holding
// the target rank, and stops once a bin is a single key (at most three
// passes for 32-bit keys, one when all keys are equal).
//
// One thread-block cluster of 8 CTAs does the work with no global scratch:
// each CTA histograms its eighth of the scores in shared memory (plain
// atomics; the first pass builds one histogram for both targets), the 8
// histograms are summed through distributed shared memory after a cluster
// barrier (each thread issues all its remote loads before using any), and
// every CTA finds the same bin by a block-wide scan of the totals (two bins
// per thread).  Histograms are double buffered so one cluster barrier per
// pass suffices.  The key range and the non-finite check ride on the first
// cluster barrier.  The tie pass counts
// threshold ties per thread over a contiguous range, scans them inside the
// CTA and across the 8 CTAs (again through distributed shared memory), then
// writes the levels.  Each CTA keeps its slice of keys in shared memory
// (up to 40K keys, i.e. 320K scores per cluster; beyond that the passes
// re-read them from L2).  Exact and deterministic.
#include <cooperative_groups.h>

#include "jano_common.cuh"

namespace cg = cooperative_groups;

namespace jano {
namespace {

constexpr int kCluster = 8;
constexpr int kThreads = 1024;
constexpr int kBinBits = 11;
constexpr int kBins = 1 << kBinBits;    // bins per histogram
constexpr int kMaxCachedKeys = 40 * 1024;   // keys per CTA kept in shared memory (160 KB)

// Order-preserving map float bits -> uint32 (unsigned order == float order),
// with -0 folded onto +0.
__device__ __forceinline__ uint32_t order_key(uint32_t b) {
    if (b == 0x80000000u) b = 0u;
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

struct Shared {
    // [buffer][target][bin], 32 KB.  Pass p histograms into buffer p&1; once
    // the pass's cluster barrier has passed, no peer reads buffer (p&1)^1 any
    // more, so it holds this CTA's copy of the cluster-wide totals.
    unsigned hist[2][2][kBins];
    unsigned lo[2], need[2];             // per target: bucket start (key), rank left in it
    unsigned wsum[2][32];
    unsigned ctot[2];                    // this CTA's tie counts (read by peers)
    unsigned kmin, kmax;                 // this CTA's key range (read by peers)
    int bad;
};

// Bits needed to write x (0 for x == 0).
__device__ __forceinline__ int bit_length(uint32_t x) { return x ? 32 - __clz(x) : 0; }

__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kThreads, 1)
classify_kernel(const uint32_t* __restrict__ bits, int n, long long k_static,
                long long k_active, uint8_t* __restrict__ levels, int* err) {
    __shared__ Shared sh;
    extern __shared__ uint32_t cached[];     // this CTA's order keys, when they fit
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // this CTA's slice of the scores
    const int per_cta = (n + kCluster - 1) / kCluster;
    const int lo = min(n, rank * per_cta), hi = min(n, lo + per_cta);

    const bool live0 = k_static > 0 && k_static < n;
    const bool live1 = k_active > 0 && k_active < n;

    // ---- one coalesced sweep: non-finite check, key range, keys into shared memory
    const bool use_cache = hi - lo <= kMaxCachedKeys;
    int bad = 0;
    uint32_t kmn = 0xFFFFFFFFu, kmx = 0u;
    for (int i = lo + tid; i < hi; i += kThreads) {
        const uint32_t b = __ldg(bits + i);
        bad |= (b & 0x7F800000u) == 0x7F800000u;
        const uint32_t u = order_key(b);
        kmn = min(kmn, u);
        kmx = max(kmx, u);
        if (use_cache) cached[i - lo] = u;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        kmn = min(kmn, __shfl_xor_sync(0xFFFFFFFFu, kmn, o));
        kmx = max(kmx, __shfl_xor_sync(0xFFFFFFFFu, kmx, o));
    }
    if (tid == 0) { sh.kmin = 0xFFFFFFFFu; sh.kmax = 0u; }
    __syncthreads();
    if (lane == 0) { atomicMin(&sh.kmin, kmn); atomicMax(&sh.kmax, kmx); }
    bad = __syncthreads_or(bad);
    // key of element i (lo <= i < hi)
    auto key = [&](int i) { return use_cache ? cached[i - lo] : order_key(__ldg(bits + i)); };
    if (tid == 0) {
        sh.bad = bad;
        sh.need[0] = (unsigned)(k_static < 0 ? 0 : (k_static > n ? n : k_static));
        sh.need[1] = (unsigned)(k_active < 0 ? 0 : (k_active > n ? n : k_active));
    }
    cluster.sync();
    int any_bad = 0;
    uint32_t gmin = 0xFFFFFFFFu, gmax = 0u;
    for (int r = 0; r < kCluster; ++r) {
        const Shared* peer = cluster.map_shared_rank(&sh, r);
        any_bad |= peer->bad;
        gmin = min(gmin, peer->kmin);
        gmax = max(gmax, peer->kmax);
    }
    if (any_bad) {
        if (rank == 0 && tid == 0) raise_error(err, JANO_ENONFINITE);
        cluster.sync();            // peers may still be reading our flags
        return;
    }

    // ---- radix select over the key range [gmin, gmax], most significant digit
    // first.  Each pass splits the current bucket of both targets into 2048
    // bins of 2^shift keys; the first pass's bucket is the whole range (so the
    // bins spread over the keys that occur, which keeps atomics apart), and
    // the passes stop once a bin is a single key.
    int shift = max(0, bit_length(gmax - gmin) - kBinBits);
    int bucket_bits = 32;                    // width of the current buckets, log2
    if (tid == 0) sh.lo[0] = sh.lo[1] = gmin;
    for (int pass = 0;; ++pass) {
        const int buf = pass & 1;
        const bool one = pass == 0;          // one histogram serves both targets
        const int nh = one ? 1 : 2;
        for (int b = tid; b < nh * kBins; b += kThreads) (&sh.hist[buf][0][0])[b] = 0u;
        __syncthreads();                     // sh.lo of the previous pass is visible too
        const uint32_t lo0 = sh.lo[0], lo1 = sh.lo[1];
        const unsigned need0 = sh.need[0], need1 = sh.need[1];
        // candidates: keys inside the target's current bucket of 2^bucket_bits keys
        const uint32_t width_m1 = bucket_bits >= 32 ? 0xFFFFFFFFu : (1u << bucket_bits) - 1u;
        for (int i = lo + tid; i < hi; i += kThreads) {
            const uint32_t u = key(i);
            if (one) {
                if (live0 || live1) atomicAdd(&sh.hist[buf][0][(u - lo0) >> shift], 1u);
            } else {
                if (live0 && u - lo0 <= width_m1) atomicAdd(&sh.hist[buf][0][(u - lo0) >> shift], 1u);
                if (live1 && u - lo1 <= width_m1) atomicAdd(&sh.hist[buf][1][(u - lo1) >> shift], 1u);
            }
        }
        cluster.sync();            // all 8 local histograms of this pass are complete
        // cluster-wide totals: every remote load of this thread issued before any is used
        {
            const unsigned* rem[kCluster];
#pragma unroll
            for (int r = 0; r < kCluster; ++r) rem[r] = cluster.map_shared_rank(&sh.hist[buf][0][0], r);
            unsigned v[4][kCluster];
#pragma unroll
            for (int k = 0; k < 4; ++k)
                if (k < 2 * nh) {
#pragma unroll
                    for (int r = 0; r < kCluster; ++r) v[k][r] = rem[r][tid + k * kThreads];
                }
#pragma unroll
            for (int k = 0; k < 4; ++k)
                if (k < 2 * nh) {
                    unsigned t = 0;
#pragma unroll
                    for (int r = 0; r < kCluster; ++r) t += v[k][r];
                    (&sh.hist[buf ^ 1][0][0])[tid + k * kThreads] = t;
                }
        }
        __syncthreads();
        // block-wide scan of the totals, two bins per thread, both targets at once
        const unsigned* h0 = sh.hist[buf ^ 1][0];
        const unsigned* h1 = sh.hist[buf ^ 1][one ? 0 : 1];
        const unsigned a0 = h0[2 * tid], b0 = h0[2 * tid + 1];
        const unsigned a1 = h1[2 * tid], b1 = h1[2 * tid + 1];
        unsigned x0 = a0 + b0, x1 = a1 + b1;
        unsigned i0 = x0, i1 = x1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned y0 = __shfl_up_sync(0xFFFFFFFFu, i0, o);
            const unsigned y1 = __shfl_up_sync(0xFFFFFFFFu, i1, o);
            if (lane >= o) { i0 += y0; i1 += y1; }
        }
        if (lane == 31) { sh.wsum[0][warp] = i0; sh.wsum[1][warp] = i1; }
        __syncthreads();
        if (warp == 0) {
            const unsigned w0 = sh.wsum[0][lane], w1 = sh.wsum[1][lane];
            unsigned j0 = w0, j1 = w1;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned y0 = __shfl_up_sync(0xFFFFFFFFu, j0, o);
                const unsigned y1 = __shfl_up_sync(0xFFFFFFFFu, j1, o);
                if (lane >= o) { j0 += y0; j1 += y1; }
            }
            __syncwarp();
            sh.wsum[0][lane] = j0 - w0;       // exclusive prefix of the warp totals
            sh.wsum[1][lane] = j1 - w1;
        }
        __syncthreads();
        // the one thread whose two bins hold rank `need` narrows the bucket
        const unsigned e0 = sh.wsum[0][warp] + i0 - x0, e1 = sh.wsum[1][warp] + i1 - x1;
        if (live0 && e0 <= need0 && need0 < e0 + x0) {
            const bool first = need0 < e0 + a0;
            sh.lo[0] = lo0 + ((uint32_t)(2 * tid + (first ? 0 : 1)) << shift);
            sh.need[0] = need0 - e0 - (first ? 0u : a0);
        }
        if (live1 && e1 <= need1 && need1 < e1 + x1) {
            const bool first = need1 < e1 + a1;
            sh.lo[1] = lo1 + ((uint32_t)(2 * tid + (first ? 0 : 1)) << shift);
            sh.need[1] = need1 - e1 - (first ? 0u : a1);
        }
        if (shift == 0) break;              // the bucket is one key: its value is lo
        bucket_bits = shift;
        shift = max(0, shift - kBinBits);
    }
    __syncthreads();

    // ---- ties at the threshold values, resolved by block index
    const uint32_t v0 = sh.lo[0], v1 = sh.lo[1];
    const unsigned need0 = sh.need[0], need1 = sh.need[1];
    const int per_thr = (hi - lo + kThreads - 1) / kThreads;
    const int tlo = min(hi, lo + tid * per_thr), thi = min(hi, tlo + per_thr);
    unsigned c0 = 0, c1 = 0;
    for (int i = tlo; i < thi; ++i) {
        const uint32_t u = key(i);
        c0 += live0 && u == v0;
        c1 += live1 && u == v1;
    }
    // exclusive scan of (c0, c1) over the CTA's threads
    unsigned s0 = c0, s1 = c1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned y0 = __shfl_up_sync(0xFFFFFFFFu, s0, o);
        const unsigned y1 = __shfl_up_sync(0xFFFFFFFFu, s1, o);
        if (lane >= o) { s0 += y0; s1 += y1; }
    }
    if (lane == 31) { sh.wsum[0][warp] = s0; sh.wsum[1][warp] = s1; }
    __syncthreads();
    unsigned w0 = 0, w1 = 0, t0 = 0, t1 = 0;
    for (int w = 0; w < kThreads / 32; ++w) {
        if (w < warp) { w0 += sh.wsum[0][w]; w1 += sh.wsum[1][w]; }
        t0 += sh.wsum[0][w];
        t1 += sh.wsum[1][w];
    }
    if (tid == 0) { sh.ctot[0] = t0; sh.ctot[1] = t1; }
    cluster.sync();
    unsigned b0 = 0, b1 = 0;
    for (int r = 0; r < rank; ++r) {
        b0 += cluster.map_shared_rank(sh.ctot, r)[0];
        b1 += cluster.map_shared_rank(sh.ctot, r)[1];
    }
    unsigned tie0 = b0 + w0 + s0 - c0, tie1 = b1 + w1 + s1 - c1;
    for (int i = tlo; i < thi; ++i) {
        const uint32_t u = key(i);
        const bool e0 = live0 && u == v0, e1 = live1 && u == v1;
        // rank < k_static ?  rank < k_active ?
        const bool below_s = live0 ? (u < v0 || (e0 && tie0 < need0)) : (k_static >= n);
        const bool below_a = live1 ? (u < v1 || (e1 && tie1 < need1)) : (k_active >= n);
        levels[i] = below_s ? 1 : (below_a ? 2 : 3);
        tie0 += e0;
        tie1 += e1;
    }
    cluster.sync();                // keep shared memory alive until peers are done
}

}  // namespace

cudaError_t launch_classify(const float* scores, int n, long long k_static,
                            long long k_active, uint8_t* levels, int* err,
                            cudaStream_t st) {
    const int per_cta = (n + kCluster - 1) / kCluster;
    const size_t smem = per_cta <= kMaxCachedKeys ? (size_t)per_cta * 4 : 0;
    static DeviceOnce opted_in;   // per-device shared-memory opt-in
    int dev = 0;
    cudaGetDevice(&dev);
    if (!opted_in.done(dev)) {
        cudaError_t e = cudaFuncSetAttribute(classify_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kMaxCachedKeys * 4);
        if (e != cudaSuccess) return e;
        opted_in.mark(dev);
    }
    classify_kernel<<<kCluster, kThreads, smem, st>>>(reinterpret_cast<const uint32_t*>(scores), n,
                                                      k_static, k_active, levels, err);
    return cudaGetLastError();
}

}  // namespace jano
