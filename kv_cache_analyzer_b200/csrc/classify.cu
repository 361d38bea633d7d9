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
// cluster barrier.
//
// After the first pass the two target buckets usually hold few keys, so
// every CTA copies the candidates of all 8 CTAs (keys with their element
// indices, through distributed shared memory: one more cluster barrier) and
// finishes the select on them alone; among the candidates equal to the
// threshold key it takes the one whose index has the remaining rank, so the
// threshold element itself -- key and index -- is known, and every CTA
// writes its levels by comparing (score, index) pairs with it: no further
// cluster-wide pass.  Small exchanges (key ranges, candidate counts) are
// written into every CTA's shared memory before a cluster barrier rather
// than read from the peers after it.  When a bucket
// holds more keys than the buffers (many equal scores), every CTA takes the
// other route: the cluster-wide passes continue, and a tie pass counts
// threshold ties per thread over a contiguous range, scans them inside the
// CTA and across the 8 CTAs (again through distributed shared memory), then
// writes the levels.  Each CTA keeps its slice of keys in shared memory
// (up to 24K keys, i.e. 192K scores per cluster; beyond that the passes
// re-read them from L2).  Exact and deterministic.
#include <cooperative_groups.h>

#include "jano_common.cuh"

namespace cg = cooperative_groups;

namespace jano {
namespace {

constexpr int kCluster = 8;
constexpr int kThreads = 1024;
constexpr int kWarpsC = kThreads / 32;
constexpr int kBinBits = 11;
constexpr int kBins = 1 << kBinBits;    // bins per histogram
constexpr int kMaxCachedKeys = 24 * 1024;   // keys per CTA kept in shared memory (96 KB)
constexpr int kCand = 1024;                 // candidates per target a CTA may hold
constexpr int kGather = 4096;               // candidates per target of the whole cluster
// dynamic shared memory after the key cache: [2][kCand] keys and indices,
// then [2][kGather] keys and indices
constexpr size_t kCandBytes = (size_t)(4 * kCand + 4 * kGather) * 4;

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
    unsigned ithr[2];                    // index of each target's threshold element
    int bad;
    // filled by every CTA of the cluster (remote stores before a cluster
    // barrier), so that reading them needs no remote load
    unsigned xmin[kCluster], xmax[kCluster];   // each CTA's key range
    int xbad[kCluster];                        // each CTA's non-finite flag
    unsigned xc0[kCluster], xc1[kCluster];     // each CTA's candidate counts
    int xover[kCluster];                       // each CTA's candidates overflowed
    unsigned wtot[2];                          // block totals of a scan
};

// Bits needed to write x (0 for x == 0).
__device__ __forceinline__ int bit_length(uint32_t x) { return x ? 32 - __clz(x) : 0; }



// kCache: the CTA's keys are kept in shared memory (slices of up to
// kMaxCachedKeys); otherwise every pass re-reads the scores.  A template
// flag, so that the cached form never issues the global loads.
template <bool kCache>
__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kThreads, 1)
classify_kernel(const uint32_t* __restrict__ bits, int n, long long k_static,
                long long k_active, uint8_t* __restrict__ levels, int* err) {
    __shared__ Shared sh;
    extern __shared__ uint32_t cached[];     // this CTA's order keys, when they fit
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // first half of a cluster barrier: before this CTA's first remote store
    // (below) every CTA of the cluster has started
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");

    // this CTA's slice of the scores (a multiple of 4 elements, so that slices
    // start 4-aligned)
    const int per_cta = ((n + kCluster - 1) / kCluster + 3) / 4 * 4;
    const int lo = min(n, rank * per_cta), hi = min(n, lo + per_cta);

    const bool live0 = k_static > 0 && k_static < n;
    const bool live1 = k_active > 0 && k_active < n;

    // ---- one coalesced sweep: non-finite check, key range, keys into shared memory
    // the same layout in every CTA (peers address each other's buffers by offset)
    constexpr bool use_cache = kCache;
    int bad = 0;
    uint32_t kmn = 0xFFFFFFFFu, kmx = 0u;
    // eight loads per thread in flight before any is used (the scores come
    // from DRAM or L2, and this sweep is on the critical path)
    for (int i0 = lo + tid; i0 < hi; i0 += 8 * kThreads) {
        uint32_t b[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int i = i0 + j * kThreads;
            b[j] = i < hi ? __ldg(bits + i) : 0u;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int i = i0 + j * kThreads;
            if (i < hi) {
                bad |= (b[j] & 0x7F800000u) == 0x7F800000u;
                const uint32_t u = order_key(b[j]);
                kmn = min(kmn, u);
                kmx = max(kmx, u);
                if constexpr (kCache) cached[i - lo] = u;
            }
        }
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
    auto key = [&](int i) -> uint32_t {
        if constexpr (kCache) return cached[i - lo];
        else return order_key(__ldg(bits + i));
    };
    if (tid == 0) {
        sh.need[0] = (unsigned)(k_static < 0 ? 0 : (k_static > n ? n : k_static));
        sh.need[1] = (unsigned)(k_active < 0 ? 0 : (k_active > n ? n : k_active));
    }
    // this CTA's flag and key range into slot `rank` of every CTA
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
    if (tid < kCluster) {
        Shared* peer = cluster.map_shared_rank(&sh, tid);
        peer->xbad[rank] = bad;
        peer->xmin[rank] = sh.kmin;
        peer->xmax[rank] = sh.kmax;
    }
    cluster.sync();
    int any_bad = 0;
    uint32_t gmin = 0xFFFFFFFFu, gmax = 0u;
#pragma unroll
    for (int r = 0; r < kCluster; ++r) {
        any_bad |= sh.xbad[r];
        gmin = min(gmin, sh.xmin[r]);
        gmax = max(gmax, sh.xmax[r]);
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
    // Block-wide scan of two 2048-bin histograms (two bins per thread, both
    // targets at once); the one thread whose bins hold rank `need` of a target
    // narrows that target's bucket to the bin (lo += bin << shift) and leaves
    // the rank inside it.  Ends with every thread past the update.
    auto scan_pick = [&](const unsigned* h0, const unsigned* h1, uint32_t lo0, uint32_t lo1,
                         unsigned need0, unsigned need1, int shift) {
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
        __syncthreads();
    };

    int pass = 0;
    bool finished = false;
    auto cluster_pass = [&]() {
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
        scan_pick(sh.hist[buf ^ 1][0], sh.hist[buf ^ 1][one ? 0 : 1], lo0, lo1, need0, need1, shift);
        if (shift == 0) {                   // the bucket is one key: its value is lo
            finished = true;
        } else {
            bucket_bits = shift;
            shift = max(0, shift - kBinBits);
        }
        ++pass;
        __syncthreads();
    };
    // Candidates of the first pass's buckets, gathered from all CTAs, and
    // the rest of the select on them alone (see below); false when they do
    // not fit the buffers.
    const int cache_words = use_cache ? per_cta : 0;
    uint32_t* cu = cached + cache_words;         // [2][kCand] this CTA's candidate keys
    uint32_t* ci = cu + 2 * kCand;               // [2][kCand] and their element indices
    uint32_t* gu = ci + 2 * kCand;               // [2][kGather] the cluster's candidates
    uint32_t* gi = gu + 2 * kGather;
    auto gather_select = [&](uint32_t (&ithr)[2]) -> bool {
        const uint32_t lo0 = sh.lo[0], lo1 = sh.lo[1];
        const uint32_t wm1 = bucket_bits >= 32 ? 0xFFFFFFFFu : (1u << bucket_bits) - 1u;
        // this CTA's candidates: each warp sweeps a contiguous chunk of the
        // CTA's range twice (count, then write at running offsets from its
        // base), one block scan of the warp counts between; no atomics
        const unsigned lt = (1u << lane) - 1u;
        const int wchunk = (hi - lo + 32 * kWarpsC - 1) / (32 * kWarpsC) * 32;
        const int wlo = min(hi, lo + warp * wchunk), whi = min(hi, wlo + wchunk);
        unsigned n0 = 0, n1 = 0;
        for (int i = wlo + lane; i - lane < whi; i += 32) {
            const uint32_t u = i < whi ? key(i) : 0u;
            n0 += __popc(__ballot_sync(0xFFFFFFFFu, i < whi && live0 && u - lo0 <= wm1));
            n1 += __popc(__ballot_sync(0xFFFFFFFFu, i < whi && live1 && u - lo1 <= wm1));
        }
        if (lane == 0) { sh.wsum[0][warp] = n0; sh.wsum[1][warp] = n1; }
        __syncthreads();
        if (warp == 0) {                     // exclusive prefix of the warp counts, and the total
            const unsigned a = sh.wsum[0][lane], b = sh.wsum[1][lane];
            unsigned ia = a, ib = b;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned ya = __shfl_up_sync(0xFFFFFFFFu, ia, o);
                const unsigned yb = __shfl_up_sync(0xFFFFFFFFu, ib, o);
                if (lane >= o) { ia += ya; ib += yb; }
            }
            __syncwarp();
            sh.wsum[0][lane] = ia - a;
            sh.wsum[1][lane] = ib - b;
            if (lane == 31) { sh.wtot[0] = ia; sh.wtot[1] = ib; }
        }
        __syncthreads();
        if (sh.wtot[0] <= (unsigned)kCand && sh.wtot[1] <= (unsigned)kCand) {
            unsigned p0 = sh.wsum[0][warp], p1 = sh.wsum[1][warp];
            for (int i = wlo + lane; i - lane < whi; i += 32) {
                const uint32_t u = i < whi ? key(i) : 0u;
                const bool m0 = i < whi && live0 && u - lo0 <= wm1;
                const bool m1 = i < whi && live1 && u - lo1 <= wm1;
                const unsigned b0 = __ballot_sync(0xFFFFFFFFu, m0), b1 = __ballot_sync(0xFFFFFFFFu, m1);
                if (m0) { const unsigned q = p0 + __popc(b0 & lt); cu[q] = u; ci[q] = (uint32_t)i; }
                if (m1) { const unsigned q = p1 + __popc(b1 & lt); cu[kCand + q] = u; ci[kCand + q] = (uint32_t)i; }
                p0 += __popc(b0);
                p1 += __popc(b1);
            }
        }
        const unsigned t0 = sh.wtot[0], t1 = sh.wtot[1];
        const bool fits = t0 <= (unsigned)kCand && t1 <= (unsigned)kCand;
        // this CTA's counts into slot `rank` of every CTA
        if (tid < kCluster) {
            Shared* peer = cluster.map_shared_rank(&sh, tid);
            peer->xc0[rank] = t0;
            peer->xc1[rank] = t1;
            peer->xover[rank] = fits ? 0 : 1;
        }
        cluster.sync();            // every CTA's list and counts are complete
        unsigned cnt0[kCluster], cnt1[kCluster], T0 = 0, T1 = 0;
        int over = 0;
#pragma unroll
        for (int r = 0; r < kCluster; ++r) {
            cnt0[r] = sh.xc0[r];
            cnt1[r] = sh.xc1[r];
            over |= sh.xover[r];
            T0 += cnt0[r];
            T1 += cnt1[r];
        }
        if (over || T0 > (unsigned)kGather || T1 > (unsigned)kGather) return false;   // same in every CTA
        // gather: CTA r's list follows those of CTAs 0..r-1; each thread takes
        // entries k = tid, tid + 1024, ... of the joined list, so its remote
        // loads do not wait on one another
        auto gather_list = [&](int t, const unsigned (&cnt)[kCluster], unsigned total) {
#pragma unroll 4
            for (unsigned k = tid; k < total; k += kThreads) {
                unsigned r = 0, base_r = 0, pre = 0;
#pragma unroll
                for (int q = 0; q < kCluster; ++q) {     // source CTA of entry k
                    const unsigned next = pre + cnt[q];
                    if (k >= next) { r = q + 1; base_r = next; }
                    pre = next;
                }
                const unsigned j = t * kCand + (k - base_r);
                gu[t * kGather + k] = cluster.map_shared_rank(cu, r)[j];
                gi[t * kGather + k] = cluster.map_shared_rank(ci, r)[j];
            }
        };
        gather_list(0, cnt0, T0);
        gather_list(1, cnt1, T1);
        __syncthreads();
        // the rest of the radix select on the gathered candidates, in this CTA
        int bits = bucket_bits;
        for (;;) {
            const int sft = max(0, bits - kBinBits);
            const uint32_t l0 = sh.lo[0], l1 = sh.lo[1];
            const unsigned nd0 = sh.need[0], nd1 = sh.need[1];
            const uint32_t bm1 = bits >= 32 ? 0xFFFFFFFFu : (1u << bits) - 1u;
            for (int b = tid; b < 2 * kBins; b += kThreads) (&sh.hist[0][0][0])[b] = 0u;
            __syncthreads();               // also: the gathered lists are complete
            for (unsigned j = tid; j < T0; j += kThreads) {
                const uint32_t u = gu[j];
                if (u - l0 <= bm1) atomicAdd(&sh.hist[0][0][(u - l0) >> sft], 1u);
            }
            for (unsigned j = tid; j < T1; j += kThreads) {
                const uint32_t u = gu[kGather + j];
                if (u - l1 <= bm1) atomicAdd(&sh.hist[0][1][(u - l1) >> sft], 1u);
            }
            __syncthreads();
            scan_pick(sh.hist[0][0], sh.hist[0][1], l0, l1, nd0, nd1, sft);
            if (sft == 0) break;           // the bucket is one key: its value is sh.lo
            bits = sft;
        }
        // ties at the threshold key: the need-th smallest index among the
        // candidates equal to it (usually there is one)
        const uint32_t v[2] = {sh.lo[0], sh.lo[1]};
        const unsigned nd[2] = {sh.need[0], sh.need[1]};
        const unsigned T[2] = {T0, T1};
        uint32_t* tl = &sh.hist[1][0][0];    // tie list, up to 4096 indices (the histograms are done)
        for (int t = 0; t < 2; ++t) {
            const bool live = t ? live1 : live0;
            if (tid == 0) sh.wtot[0] = 0u;
            __syncthreads();
            for (unsigned j = tid; j < T[t]; j += kThreads)
                if (gu[t * kGather + j] == v[t]) tl[atomicAdd(&sh.wtot[0], 1u)] = gi[t * kGather + j];
            __syncthreads();
            const unsigned c = sh.wtot[0];
            for (unsigned e = tid; live && e < c; e += kThreads) {
                const uint32_t me = tl[e];
                unsigned r = 0;
                for (unsigned f = 0; f < c; ++f) r += tl[f] < me;
                if (r == nd[t]) sh.ithr[t] = me;
            }
            __syncthreads();
        }
        ithr[0] = sh.ithr[0];
        ithr[1] = sh.ithr[1];
        return true;
    };

    cluster_pass();                          // pass 0 over every key

    // ---- after the first pass the target buckets usually hold few keys:
    // every CTA gathers the candidates of all 8 CTAs (keys with their indices) through
    // distributed shared memory and finishes the select alone, then resolves
    // ties by index among those candidates, so no further cluster-wide pass
    // and no cross-CTA tie scan is needed.  When a bucket holds more keys
    // than the gather buffers (many equal scores), the cluster-wide passes
    // and the tie scan below run instead; the choice is the same in all CTAs.
    bool composite = false;
    uint32_t i_thr[2] = {0u, 0u};            // the threshold element's index per target
    if (!finished) composite = gather_select(i_thr);
    if (!composite) {
        while (!finished) cluster_pass();
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
    } else {
        // rank < k_static  <=>  (key, index) < the threshold element of target 0
        const uint32_t v0 = sh.lo[0], v1 = sh.lo[1];
        auto level_of = [&](int i, uint32_t u) -> uint8_t {
            const bool below_s = live0 ? (u < v0 || (u == v0 && (uint32_t)i < i_thr[0])) : (k_static >= n);
            const bool below_a = live1 ? (u < v1 || (u == v1 && (uint32_t)i < i_thr[1])) : (k_active >= n);
            return below_s ? 1 : (below_a ? 2 : 3);
        };
        if (kCache && (reinterpret_cast<uintptr_t>(levels) & 3u) == 0) {
            // four consecutive elements per thread: one 16-byte key load, one 4-byte store
            for (int i4 = lo + 4 * tid; i4 < hi; i4 += 4 * kThreads) {
                const uint4 k4 = *reinterpret_cast<const uint4*>(cached + (i4 - lo));
                const uint8_t l0 = level_of(i4, k4.x), l1 = level_of(i4 + 1, k4.y);
                const uint8_t l2 = level_of(i4 + 2, k4.z), l3 = level_of(i4 + 3, k4.w);
                if (i4 + 3 < hi) {
                    *reinterpret_cast<uchar4*>(levels + i4) = make_uchar4(l0, l1, l2, l3);
                } else {
                    levels[i4] = l0;
                    if (i4 + 1 < hi) levels[i4 + 1] = l1;
                    if (i4 + 2 < hi) levels[i4 + 2] = l2;
                }
            }
        } else {
            for (int i = lo + tid; i < hi; i += kThreads) levels[i] = level_of(i, key(i));
        }
    }
    cluster.sync();                // keep shared memory alive until peers are done
}

}  // namespace

cudaError_t launch_classify(const float* scores, int n, long long k_static,
                            long long k_active, uint8_t* levels, int* err,
                            cudaStream_t st) {
    const int per_cta = ((n + kCluster - 1) / kCluster + 3) / 4 * 4;    // as in the kernel
    const size_t smem = (per_cta <= kMaxCachedKeys ? (size_t)per_cta * 4 : 0) + kCandBytes;
    static DeviceOnce opted_in;   // per-device shared-memory opt-in
    int dev = 0;
    cudaGetDevice(&dev);
    if (!opted_in.done(dev)) {
        cudaError_t e = cudaFuncSetAttribute(classify_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)(kMaxCachedKeys * 4 + kCandBytes));
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(classify_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)kCandBytes);
        if (e != cudaSuccess) return e;
        opted_in.mark(dev);
    }
    const uint32_t* keys = reinterpret_cast<const uint32_t*>(scores);
    if (per_cta <= kMaxCachedKeys)
        classify_kernel<true><<<kCluster, kThreads, smem, st>>>(keys, n, k_static, k_active, levels, err);
    else
        classify_kernel<false><<<kCluster, kThreads, smem, st>>>(keys, n, k_static, k_active, levels, err);
    return cudaGetLastError();
}

}  // namespace jano

