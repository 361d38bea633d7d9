// classify.cu -- three-level split of block scores (Jano pages: nl technical
// summary, Methodologie 1 "Resultaat": Level 1 Static, 2 Moderate, 3 Active;
// zh 2.2 item 1).
//
// Blocks are ranked by the key (score, block index).  A block is Static when
// its rank is below k_static = n_S and Active when its rank is at least
// k_active = n - n_A.  Instead of sorting, the kernel finds, for each of the
// two rank thresholds, the threshold element -- the (score, block index)
// pair at that rank -- by a histogram select, then writes each block's level
// by comparing its pair with the two threshold pairs.
//
// One thread-block cluster does the work with no global scratch: 16 CTAs
// where the device can run such a cluster (a non-portable size; B200 can),
// else 8.  Each CTA keeps its slice of the scores as order keys in shared
// memory (up to 24K keys per CTA; beyond that the passes re-read them from
// L2).  Small exchanges (key ranges, candidate counts) are written into
// every CTA's shared memory before a cluster barrier rather than read from
// the peers after it; histograms are double buffered so one cluster barrier
// per pass suffices.
//
// First pass.  When the scores span a finite, non-empty range, it bins the
// float values: 2048 equal-width bins between the smallest and the largest
// score (bins of the order keys would crowd into the few exponents that
// occur).  Each CTA histograms its slice with shared-memory atomics (one
// histogram serves both targets), the histograms are summed through
// distributed shared memory in rank order, and every CTA finds the same bin
// of each target, and the rank left inside it, by a block-wide scan.
//
// Candidates.  Each CTA lists its keys in the two target bins (one sweep,
// slots taken per warp with one shared atomic; the order of a list does not
// matter), every CTA copies the lists of the whole cluster (keys with their
// element indices; one more cluster barrier), and with at most 512
// candidates per target each candidate's rank in its bin is counted directly
// against all the others in (key, index) order, the candidates dealt to the
// CTAs round-robin; the one whose rank is the rank left in the bin is the
// threshold element, which its CTA writes into every CTA before a cluster
// barrier.  With more candidates every CTA runs radix passes over the
// gathered list (2048 bins of the order keys per pass) and takes, among the
// candidates equal to the threshold key, the index of the remaining rank.
// Either way the threshold element itself -- key and index -- is known, and
// every CTA writes its levels by comparing (score, index) pairs with it.
//
// Fallback.  When a bin holds more keys than the gather buffers (many equal
// scores), or the range is empty, the select runs on the order keys: radix
// passes over the key range [min, max] (each splits the current bucket of
// both targets into 2048 bins of 2^shift keys, and they stop once a bin is a
// single key), then a tie pass counts threshold ties per thread over a
// contiguous range, scans them inside the CTA and across the cluster, and
// writes the levels.  Exact and deterministic.
#include <cooperative_groups.h>

#include <atomic>
#include <cfloat>

#include "jano_common.cuh"

namespace cg = cooperative_groups;

namespace jano {
namespace {

constexpr int kMaxCluster = 16;       // CTAs per cluster: 16 where the device runs such clusters, else 8
// 8: always the portable 8-CTA cluster (a build switch that keeps that form tested)
#ifndef JANO_CLASSIFY_CLUSTER
#define JANO_CLASSIFY_CLUSTER 0
#endif
constexpr int kThreads = 1024;
constexpr int kBinBits = 11;
constexpr int kBins = 1 << kBinBits;    // bins per histogram
constexpr int kMaxCachedKeys = 24 * 1024;   // keys per CTA kept in shared memory (96 KB)
constexpr int kCand = 1024;                 // candidates per target a CTA may hold
constexpr int kGather = 4096;               // candidates per target of the whole cluster
constexpr int kDirect = 512;                // up to this many per target: select by direct rank
// dynamic shared memory after the key cache: [2][kCand] keys and indices,
// then [2][kGather] keys and indices
constexpr size_t kCandBytes = (size_t)(4 * kCand + 4 * kGather) * 4;

// Order-preserving map float bits -> uint32 (unsigned order == float order),
// with -0 folded onto +0.
__device__ __forceinline__ uint32_t order_key(uint32_t b) {
    if (b == 0x80000000u) b = 0u;
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// 32-bit load from this CTA's shared memory by its shared-window address
// (the candidate lists are reached through pointers whose address space the
// compiler does not track into the loops below).
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

// The float whose order key is u (the inverse of order_key; -0 comes back as +0).
__device__ __forceinline__ float key_value(uint32_t u) {
    return __uint_as_float((u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u);
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
    unsigned vb[2];                      // each target's bin of the value-domain first pass
    unsigned smin, smax;                 // key range of the sample (the same in every CTA)
    unsigned own[kBins / 8];             // this CTA's share of the first pass's cluster histogram
    int bad;
    // filled by every CTA of the cluster (remote stores before a cluster
    // barrier), so that reading them needs no remote load
    unsigned xmin[kMaxCluster], xmax[kMaxCluster];   // each CTA's key range
    int xbad[kMaxCluster];                           // each CTA's non-finite flag
    unsigned xc0[kMaxCluster], xc1[kMaxCluster];     // each CTA's candidate counts
    int xover[kMaxCluster];                          // each CTA's candidates overflowed
    unsigned wtot[2];                          // block totals of a scan
};

// Bits needed to write x (0 for x == 0).
__device__ __forceinline__ int bit_length(uint32_t x) { return x ? 32 - __clz(x) : 0; }



// kCache: the CTA's keys are kept in shared memory (slices of up to
// kMaxCachedKeys); otherwise every pass re-reads the scores.  A template
// flag, so that the cached form never issues the global loads.
template <bool kCache, int kCluster>
__global__ void __launch_bounds__(kThreads, 1)
classify_kernel(const uint32_t* __restrict__ bits, int n, long long k_static,
                long long k_active, uint8_t* __restrict__ levels, int* err) {
    __shared__ Shared sh;
    extern __shared__ uint32_t cached[];     // this CTA's order keys, when they fit
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int kOwn = kBins / kCluster;   // bins of the value pass's histogram each CTA totals
    for (int b = tid; b < kOwn; b += kThreads) sh.own[b] = 0u;
    // first half of a cluster barrier (release): before this CTA's first
    // remote access (below) every CTA of the cluster has started and zeroed
    // its share of the histogram
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");

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
    // sixteen loads per thread in flight before any is used (the scores come
    // from DRAM or L2, and this sweep is on the critical path): one round
    // trip for up to 16K keys per CTA
    constexpr int kBatch = kCluster >= 16 ? 8 : 16;
    // one key of a strided sample of the whole array, the same in every CTA:
    // its range sets the bins of the value-domain first pass
    const uint32_t sbits = n > 0 ? __ldg(bits + (int)(((long long)tid * n) / kThreads)) : 0u;
    for (int i0 = lo + tid; i0 < hi; i0 += kBatch * kThreads) {
        uint32_t b[kBatch];
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
            const int i = i0 + j * kThreads;
            b[j] = i < hi ? __ldg(bits + i) : 0u;
        }
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
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
    uint32_t smn = n > 0 ? order_key(sbits) : 0xFFFFFFFFu, smx = n > 0 ? order_key(sbits) : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        kmn = min(kmn, __shfl_xor_sync(0xFFFFFFFFu, kmn, o));
        kmx = max(kmx, __shfl_xor_sync(0xFFFFFFFFu, kmx, o));
        smn = min(smn, __shfl_xor_sync(0xFFFFFFFFu, smn, o));
        smx = max(smx, __shfl_xor_sync(0xFFFFFFFFu, smx, o));
    }
    if (tid == 0) { sh.kmin = sh.smin = 0xFFFFFFFFu; sh.kmax = sh.smax = 0u; }
    __syncthreads();
    if (lane == 0) {
        atomicMin(&sh.kmin, kmn); atomicMax(&sh.kmax, kmx);
        atomicMin(&sh.smin, smn); atomicMax(&sh.smax, smx);
    }
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
    // this CTA's flag and key range into slot `rank` of every CTA; they are
    // read after the next cluster barrier
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
    if (tid < kCluster) {
        Shared* peer = cluster.map_shared_rank(&sh, tid);
        peer->xbad[rank] = bad;
        peer->xmin[rank] = sh.kmin;
        peer->xmax[rank] = sh.kmax;
    }
    const unsigned need_init0 = (unsigned)(k_static < 0 ? 0 : (k_static > n ? n : k_static));
    const unsigned need_init1 = (unsigned)(k_active < 0 ? 0 : (k_active > n ? n : k_active));
    // The first pass bins the float values rather than their order keys when
    // the sample spans a finite, non-empty range: 2048 equal-width bins over
    // the sample's range follow the values' spread, where bins of the order
    // keys crowd into the few exponents that occur (a field of mixed signs
    // fills a few hundred of them); values outside the sample's range fall
    // into the end bins.  The bin of a value is a monotone function of it,
    // computed the same way by every thread of every CTA, so a target's rank
    // falls in one bin and the rank left inside it is exact.  Its candidates
    // then go to the gather below; should they not fit, the select starts
    // over on the order keys.  Otherwise the first pass bins the order keys
    // over the cluster's key range, which takes one more cluster barrier.
    const float xlo = key_value(sh.smin), xhi = key_value(sh.smax);
    const float span = xhi - xlo;
    const float vscale = (float)kBins / span;
    bool vmode = sh.smax > sh.smin && span > 0.f && span <= FLT_MAX && vscale > 0.f && vscale <= FLT_MAX;
    auto vbin = [&](uint32_t u) -> unsigned {
        return (unsigned)min(kBins - 1, max(0, __float2int_rz((key_value(u) - xlo) * vscale)));
    };
    int any_bad = 0;
    uint32_t gmin = 0xFFFFFFFFu, gmax = 0u;
    auto read_exchange = [&]() {
#pragma unroll
        for (int r = 0; r < kCluster; ++r) {
            any_bad |= sh.xbad[r];
            gmin = min(gmin, sh.xmin[r]);
            gmax = max(gmax, sh.xmax[r]);
        }
    };
    int shift = 0;
    int bucket_bits = 32;                    // width of the current buckets, log2
    if (!vmode) {
        cluster.sync();                      // the key ranges and flags have arrived
        read_exchange();
        if (any_bad) {
            if (rank == 0 && tid == 0) raise_error(err, JANO_ENONFINITE);
            cluster.sync();                  // peers may still be reading our flags
            return;
        }
        // radix passes over the key range [gmin, gmax], most significant digit
        // first; the first pass's bucket is the whole range
        shift = max(0, bit_length(gmax - gmin) - kBinBits);
        if (tid == 0) sh.lo[0] = sh.lo[1] = gmin;
    }
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
            sh.vb[0] = 2u * tid + (first ? 0u : 1u);
            sh.lo[0] = lo0 + ((uint32_t)(2 * tid + (first ? 0 : 1)) << shift);
            sh.need[0] = need0 - e0 - (first ? 0u : a0);
        }
        if (live1 && e1 <= need1 && need1 < e1 + x1) {
            const bool first = need1 < e1 + a1;
            sh.vb[1] = 2u * tid + (first ? 0u : 1u);
            sh.lo[1] = lo1 + ((uint32_t)(2 * tid + (first ? 0 : 1)) << shift);
            sh.need[1] = need1 - e1 - (first ? 0u : a1);
        }
        __syncthreads();
    };

    int pass = 0;
    bool finished = false;
    bool fresh = true;                       // the next pass is the first over its range
    auto cluster_pass = [&]() {
        const int buf = pass & 1;
        const bool one = fresh;              // one histogram serves both targets
        const int nh = one ? 1 : 2;
        for (int b = tid; b < nh * kBins; b += kThreads) (&sh.hist[buf][0][0])[b] = 0u;
        __syncthreads();                     // sh.lo of the previous pass is visible too
        const uint32_t lo0 = sh.lo[0], lo1 = sh.lo[1];
        const unsigned need0 = sh.need[0], need1 = sh.need[1];
        // candidates: keys inside the target's current bucket of 2^bucket_bits keys
        const uint32_t width_m1 = bucket_bits >= 32 ? 0xFFFFFFFFu : (1u << bucket_bits) - 1u;
        // four consecutive keys per thread and step (independent atomics)
        for (int i4 = lo + 4 * tid; i4 < hi; i4 += 4 * kThreads) {
            uint32_t uu[4];
            if (kCache && i4 + 3 < hi) {
                const uint4 k4 = *reinterpret_cast<const uint4*>(cached + (i4 - lo));
                uu[0] = k4.x; uu[1] = k4.y; uu[2] = k4.z; uu[3] = k4.w;
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q) uu[q] = i4 + q < hi ? key(i4 + q) : 0u;
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                if (i4 + q >= hi) break;
                const uint32_t u = uu[q];
                if (one) {
                    if (live0 || live1) atomicAdd(&sh.hist[buf][0][(u - lo0) >> shift], 1u);
                } else {
                    if (live0 && u - lo0 <= width_m1) atomicAdd(&sh.hist[buf][0][(u - lo0) >> shift], 1u);
                    if (live1 && u - lo1 <= width_m1) atomicAdd(&sh.hist[buf][1][(u - lo1) >> shift], 1u);
                }
            }
        }
        cluster.sync();            // all 8 local histograms of this pass are complete
        // cluster-wide totals, peers added in rank order; a thread's remote
        // loads of one bin are all in flight before any is used
#pragma unroll 1
        for (int k = 0; k < 2 * nh; ++k) {
            unsigned v[kCluster];
#pragma unroll
            for (int r = 0; r < kCluster; ++r)
                v[r] = cluster.map_shared_rank(&sh.hist[buf][0][0], r)[tid + k * kThreads];
            unsigned t = 0;
#pragma unroll
            for (int r = 0; r < kCluster; ++r) t += v[r];
            (&sh.hist[buf ^ 1][0][0])[tid + k * kThreads] = t;
        }
        __syncthreads();
        scan_pick(sh.hist[buf ^ 1][0], sh.hist[buf ^ 1][one ? 0 : 1], lo0, lo1, need0, need1, shift);
        if (shift == 0) {                   // the bucket is one key: its value is lo
            finished = true;
        } else {
            bucket_bits = shift;
            shift = max(0, shift - kBinBits);
        }
        fresh = false;
        ++pass;
        __syncthreads();
    };
    // The value-domain first pass.  Each CTA histograms its keys' value bins
    // (one histogram for both targets) and adds its counts into the owners'
    // shares: CTA r totals bins [r kOwn, (r+1) kOwn) (remote reductions into
    // distributed shared memory, integers, so the order does not matter).
    // After the cluster barrier every CTA reads the 2048 totals from the
    // owners and finds each target's bin and the rank left in it (sh.vb,
    // sh.need).  The barrier also brings the peers' flags and key ranges.
    auto value_pass = [&]() {
        for (int b = tid; b < kBins; b += kThreads) sh.hist[0][0][b] = 0u;
        __syncthreads();
        if (live0 || live1) {
            for (int i4 = lo + 4 * tid; i4 < hi; i4 += 4 * kThreads) {
                uint32_t uu[4];
                if (kCache && i4 + 3 < hi) {
                    const uint4 k4 = *reinterpret_cast<const uint4*>(cached + (i4 - lo));
                    uu[0] = k4.x; uu[1] = k4.y; uu[2] = k4.z; uu[3] = k4.w;
                } else {
#pragma unroll
                    for (int q = 0; q < 4; ++q) uu[q] = i4 + q < hi ? key(i4 + q) : 0u;
                }
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (i4 + q < hi) atomicAdd(&sh.hist[0][0][vbin(uu[q])], 1u);
            }
        }
        __syncthreads();
        const uint32_t own0 = ptx::smem_u32(&sh.own[0]);
        for (int b = tid; b < kBins; b += kThreads) {
            const unsigned v = sh.hist[0][0][b];
            if (v) ptx::red_cluster_add_u32(ptx::mapa_shared(own0 + 4u * (uint32_t)(b % kOwn), (uint32_t)(b / kOwn)), v);
        }
        cluster.sync();            // every share is complete
        for (int b = tid; b < kBins; b += kThreads)
            sh.hist[1][0][b] = ptx::ld_cluster_u32(ptx::mapa_shared(own0 + 4u * (uint32_t)(b % kOwn), (uint32_t)(b / kOwn)));
        __syncthreads();
        scan_pick(sh.hist[1][0], sh.hist[1][0], 0u, 0u, sh.need[0], sh.need[1], 0);
        fresh = false;
        pass = 1;                  // the next cluster pass, if any, histograms into buffer 1
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
        const unsigned nd0 = sh.need[0], nd1 = sh.need[1];
        const unsigned vb0 = sh.vb[0], vb1 = sh.vb[1];
        // this CTA's candidates in one sweep, each warp taking slots of its
        // lists with one shared atomic per list (the order of a list does not
        // matter to what follows); slots past kCand are counted, not written
        if (tid == 0) { sh.wtot[0] = 0u; sh.wtot[1] = 0u; }
        __syncthreads();
        const unsigned lt = (1u << lane) - 1u;
        // four consecutive keys per thread and step; a warp whose keys hold no
        // candidate (nearly all of them) moves on after one vote
        for (int base = lo; base < hi; base += 4 * kThreads) {
            const int i4 = base + 4 * tid;
            uint32_t uu[4];
            if (kCache && i4 + 3 < hi) {
                const uint4 k4 = *reinterpret_cast<const uint4*>(cached + (i4 - lo));
                uu[0] = k4.x; uu[1] = k4.y; uu[2] = k4.z; uu[3] = k4.w;
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q) uu[q] = i4 + q < hi ? key(i4 + q) : 0u;
            }
            bool m0[4], m1[4];
            bool any = false;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const bool in = i4 + q < hi;
                const unsigned vu = vmode ? vbin(uu[q]) : 0u;
                m0[q] = in && live0 && (vmode ? vu == vb0 : uu[q] - lo0 <= wm1);
                m1[q] = in && live1 && (vmode ? vu == vb1 : uu[q] - lo1 <= wm1);
                any |= m0[q] | m1[q];
            }
            if (!__any_sync(0xFFFFFFFFu, any)) continue;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const unsigned b0 = __ballot_sync(0xFFFFFFFFu, m0[q]), b1 = __ballot_sync(0xFFFFFFFFu, m1[q]);
                unsigned base0 = 0u, base1 = 0u;
                if (lane == 0) {
                    if (b0) base0 = atomicAdd(&sh.wtot[0], (unsigned)__popc(b0));
                    if (b1) base1 = atomicAdd(&sh.wtot[1], (unsigned)__popc(b1));
                }
                base0 = __shfl_sync(0xFFFFFFFFu, base0, 0);
                base1 = __shfl_sync(0xFFFFFFFFu, base1, 0);
                if (m0[q]) {
                    const unsigned slot = base0 + __popc(b0 & lt);
                    if (slot < (unsigned)kCand) { cu[slot] = uu[q]; ci[slot] = (uint32_t)(i4 + q); }
                }
                if (m1[q]) {
                    const unsigned slot = base1 + __popc(b1 & lt);
                    if (slot < (unsigned)kCand) { cu[kCand + slot] = uu[q]; ci[kCand + slot] = (uint32_t)(i4 + q); }
                }
            }
        }
        __syncthreads();
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
        unsigned T0 = 0, T1 = 0;
        int over = 0;
#pragma unroll
        for (int r = 0; r < kCluster; ++r) {
            over |= sh.xover[r];
            T0 += sh.xc0[r];
            T1 += sh.xc1[r];
        }
        if (over || T0 > (unsigned)kGather || T1 > (unsigned)kGather) return false;   // same in every CTA
        // gather: CTA r's list follows those of CTAs 0..r-1; each thread takes
        // entries k = tid, tid + 1024, ... of the joined list, so its remote
        // loads do not wait on one another
        auto gather_list = [&](int t, const unsigned* cnt, unsigned total) {
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
        gather_list(0, sh.xc0, T0);
        gather_list(1, sh.xc1, T1);
        __syncthreads();
        if (T0 <= (unsigned)kDirect && T1 <= (unsigned)kDirect) {
            // few candidates: each one's rank in its bucket by comparing its
            // (key, index) with every other candidate's; the one whose rank is
            // the rank left in the bucket is the threshold element.  The
            // candidates of the joined list (target 0's, then target 1's) are
            // dealt to the CTAs round-robin; in a CTA, P threads (a power of
            // two, an aligned lane group) share a candidate, each comparing a
            // 1/P share of the list four entries at a time, and add their
            // counts by shuffles.  The CTA that finds a threshold element
            // writes it into every CTA of the cluster, and a cluster barrier
            // publishes it.
            const unsigned Ttot = T0 + T1;
            const unsigned mine_n = Ttot > (unsigned)rank ? (Ttot - rank + kCluster - 1) / kCluster : 0u;
            unsigned P = 1;
            while (P < 32 && 2 * P * mine_n <= (unsigned)kThreads) P *= 2;
            const unsigned per_pass = kThreads / P;        // candidates per sweep of the CTA
            for (unsigned m0 = 0; m0 < mine_n; m0 += per_pass) {
                const unsigned m = m0 + (unsigned)tid / P, sub = (unsigned)tid % P;
                const unsigned c = (unsigned)rank + m * kCluster;
                const int t = c < T0 ? 0 : 1;
                const unsigned j = t ? c - T0 : c;
                const unsigned Tt = t ? T1 : T0;
                const bool mine = m < mine_n && (t ? live1 : live0);
                const uint32_t sU = (uint32_t)__cvta_generic_to_shared(gu + t * kGather);
                const uint32_t sX = (uint32_t)__cvta_generic_to_shared(gi + t * kGather);
                uint32_t u = 0u, x = 0u;
                unsigned r = 0u;
                if (mine) {
                    u = lds32(sU + 4u * j);
                    x = lds32(sX + 4u * j);
                    for (unsigned k = sub; k < Tt; k += 4 * P) {
                        uint32_t uk[4], xk[4];
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const unsigned kk = k + q * P;
                            uk[q] = kk < Tt ? lds32(sU + 4u * kk) : 0u;
                            xk[q] = kk < Tt ? lds32(sX + 4u * kk) : 0u;
                        }
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            r += (k + q * P < Tt && (uk[q] < u || (uk[q] == u && xk[q] < x))) ? 1u : 0u;
                    }
                }
                for (unsigned o = 1; o < P; o <<= 1) r += __shfl_xor_sync(0xFFFFFFFFu, r, (int)o);
                if (mine && sub == 0 && r == (t ? nd1 : nd0)) {
                    for (int q = 0; q < kCluster; ++q) {
                        Shared* peer = cluster.map_shared_rank(&sh, q);
                        peer->lo[t] = u;
                        peer->ithr[t] = x;
                    }
                }
            }
            cluster.sync();            // every CTA holds both threshold elements
            ithr[0] = sh.ithr[0];
            ithr[1] = sh.ithr[1];
            return true;
        }
        // the rest of the radix select on the gathered candidates, in this CTA
        // (after a value-domain pass the candidates span any keys: all 32 bits)
        int bits = bucket_bits;
        if (vmode) {
            if (tid == 0) sh.lo[0] = sh.lo[1] = 0u;
            bits = 32;
        }
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

    if (vmode) {
        value_pass();                        // first pass, value bins
        read_exchange();
        if (any_bad) {
            if (rank == 0 && tid == 0) raise_error(err, JANO_ENONFINITE);
            cluster.sync();                  // peers may still be reading our shares
            return;
        }
    } else {
        cluster_pass();                      // first pass, order-key bins
    }

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
        if (vmode) {
            // the value bin held more keys than the gather buffers: the select
            // starts over on the order keys (every CTA takes this branch)
            __syncthreads();
            if (tid == 0) {
                sh.lo[0] = sh.lo[1] = gmin;
                sh.need[0] = need_init0;
                sh.need[1] = need_init1;
            }
            shift = max(0, bit_length(gmax - gmin) - kBinBits);
            bucket_bits = 32;
            fresh = true;
            vmode = false;
            __syncthreads();
        }
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

namespace {
template <int kCl>
cudaError_t opt_in() {
    cudaError_t e = cudaFuncSetAttribute(classify_kernel<true, kCl>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)(kMaxCachedKeys * 4 + kCandBytes));
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(classify_kernel<false, kCl>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kCandBytes);
    if (e == cudaSuccess && kCl > 8) {
        e = cudaFuncSetAttribute(classify_kernel<true, kCl>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(classify_kernel<false, kCl>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    }
    return e;
}

template <int kCl>
cudaLaunchConfig_t cluster_config(int n, cudaStream_t st, cudaLaunchAttribute* attr, bool& cache) {
    const int per_cta = ((n + kCl - 1) / kCl + 3) / 4 * 4;    // as in the kernel
    cache = per_cta <= kMaxCachedKeys;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kCl, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = (cache ? (size_t)per_cta * 4 : 0) + kCandBytes;
    cfg.stream = st;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kCl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
}

template <int kCl>
cudaError_t launch_cluster(const uint32_t* keys, int n, long long k_static, long long k_active,
                           uint8_t* levels, int* err, cudaStream_t st) {
    cudaLaunchAttribute attr[1];
    bool cache = true;
    const cudaLaunchConfig_t cfg = cluster_config<kCl>(n, st, attr, cache);
    return cache ? cudaLaunchKernelEx(&cfg, classify_kernel<true, kCl>, keys, n, k_static, k_active, levels, err)
                 : cudaLaunchKernelEx(&cfg, classify_kernel<false, kCl>, keys, n, k_static, k_active, levels, err);
}
}  // namespace

// Clusters of 16 CTAs (twice the SMs for the sweeps over the keys) where the
// device can run one with these resources, else the portable 8; asked once
// per device.
cudaError_t launch_classify(const float* scores, int n, long long k_static,
                            long long k_active, uint8_t* levels, int* err,
                            cudaStream_t st) {
    static std::atomic<int> cluster_of[64];    // 0: not asked yet
    int dev = 0;
    cudaGetDevice(&dev);
    int cl = dev < 64 ? cluster_of[dev].load(std::memory_order_acquire) : 0;
    if (cl == 0) {
        cudaError_t e = opt_in<8>();
        if (e != cudaSuccess) return e;
        cl = 8;
        if (JANO_CLASSIFY_CLUSTER != 8 && opt_in<16>() == cudaSuccess) {
            cudaLaunchAttribute attr[1];
            bool cache = true;
            // the largest shared-memory request of the 16-CTA form (keys cached)
            cudaLaunchConfig_t cfg = cluster_config<16>(16 * kMaxCachedKeys, st, attr, cache);
            int active = 0;
            if (cudaOccupancyMaxActiveClusters(&active, classify_kernel<true, 16>, &cfg) == cudaSuccess &&
                active >= 1)
                cl = 16;
        }
        cudaGetLastError();                     // a refused query leaves no error behind
        if (dev < 64) cluster_of[dev].store(cl, std::memory_order_release);
    }
    const uint32_t* keys = reinterpret_cast<const uint32_t*>(scores);
    return cl == 16 ? launch_cluster<16>(keys, n, k_static, k_active, levels, err, st)
                    : launch_cluster<8>(keys, n, k_static, k_active, levels, err, st);
}

}  // namespace jano

