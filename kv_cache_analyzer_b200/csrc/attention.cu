// attention.cu -- active-query attention over the whole cached K/V, outputs
// scattered back to their token rows (Jano pages: nl technical summary,
// Methodologie 2 "KV Cache Mechanisme": cached K/V of frozen tokens are
// concatenated with the active queries, no position restoration, attention
// being invariant to the order of keys/values; ko 2.B; pt 2.B).
//
//   out[idx[i], h] = softmax_j(scale * q_act[i,h] . k_cache[j,h]) @ v_cache[:, h]
//
// Flash-style forward on the 5th-generation tensor cores.  One CTA per
// (pair of 128-query tiles, head); 12 warps:
//   warps 0-3, 4-7  softmax warpgroups WG0 / WG1, one per query tile:
//              thread = one query row = one TMEM lane.  Per key tile the row's
//              S (128 fp32) is read from TMEM in one round trip (setmaxnreg
//              moves registers from warps 8-11 to these two warpgroups so
//              the whole row fits), the running max
//              is kept in the log2 domain and O is rescaled in TMEM only when
//              the max grows by more than 2^8 (lazy rescale), P is written as
//              packed BF16 into the upper half of the row's S columns (keys
//              64..127 first, published on their own barrier so their P.V
//              starts while keys 0..63 are exponentiated), and at the end O
//              is normalised and stored as BF16 to out[idx[i]].
//   warp 8     TMA producer: both Q tiles once, then K_j, V_j (128 keys x d)
//              into a 4-slot shared-memory ring (128-byte swizzle, boxes of
//              64 columns); completion counted on mbarriers.
//   warp 9     allocates 512 TMEM columns; one lane issues every tcgen05.mma
//              in the ping-pong order
//                 S0_0 S1_0 | PV0_{j-1} S0_j PV1_{j-1} S1_j | ... PV0 PV1
//              so the tensor core runs one tile's MMAs while the other
//              tile's softmax runs.  S = Q K^T reads Q and K K-major from
//              smem; O += P V reads P from TMEM (A operand) and V MN-major
//              from smem.  tcgen05.commit hands S to the softmax warps and
//              frees ring slots.  Because S_i_j is issued after PV_i_{j-1},
//              the softmax that sees S_i_j may rescale O_i safely.
//   warps 10-11 idle (with 8-9 they form the warpgroup that gives up registers).
// TMEM columns: S0 [0,128) S1 [128,256) O0 [256,256+d) O1 [384,384+d);
// P_i occupies columns [64,128) of S_i.
// Every wait is bounded; on timeout the CTA records JANO_ETIMEOUT, drains its
// own copies and MMAs, frees TMEM and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <mutex>

#include "jano_common.cuh"

namespace jano {
namespace {

constexpr int BM = 128;            // queries per tile (two tiles per CTA)
constexpr int BN = 128;            // keys per tile
constexpr int kSlots = 4;          // K/V ring slots
constexpr int kThreads = 384;
// Registers per thread: at launch (384 x 168 = 64,512), then rebalanced:
// the producer / MMA warpgroup (warps 8-11) drops to kRegsIssue and the two
// softmax warpgroups rise to kRegsSoftmax, so that a softmax thread holds
// its whole 128-column S row.  2 x 128 x 208 + 128 x 80 = 63,488 of the
// 64,512, and per SM sub-partition (one warp of each warpgroup)
// 208 + 208 + 80 = 496 of 512.
constexpr int kRegsLaunch = 168;
constexpr int kRegsSoftmax = 208;
constexpr int kRegsIssue = 80;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsIssue <= kThreads * kRegsLaunch, "register split");
static_assert(2 * kRegsSoftmax + kRegsIssue <= 512, "sub-partition register file");
constexpr uint32_t kPanel = 128 * 128;   // bytes of one 128-row x 64-col BF16 panel
// d = 128 and unsplit keys take the CTA-pair kernel when this is 1
#ifndef JANO_ATTN_PAIR
#define JANO_ATTN_PAIR 0
#endif
constexpr long long kWaitLimit = 1ll << 31;  // cycles (~1 s)

template <int HD>
struct Layout {
    static constexpr int kPanels = HD / 64;
    static constexpr uint32_t kTile = kPanels * kPanel;           // Q, K or V tile bytes
    static constexpr uint32_t kQ0 = 0;
    static constexpr uint32_t kQ1 = kTile;
    static constexpr uint32_t kRing = 2 * kTile;
    static constexpr uint32_t kBar = kRing + kSlots * kTile;
    // barrier slots
    static constexpr int bQFull = 0;
    static constexpr int bFull = 1;                    // [kSlots]
    static constexpr int bEmpty = bFull + kSlots;      // [kSlots]
    static constexpr int bSFull = bEmpty + kSlots;     // [2]
    static constexpr int bPFull = bSFull + 2;          // [2] whole P written
    static constexpr int bPHalf = bPFull + 2;          // [2] P of keys 64..127 written
    static constexpr int bOFull = bPHalf + 2;          // [2]
    static constexpr int bFinal = bOFull + 2;
    static constexpr int kNumBars = bFinal + 1;
    static constexpr uint32_t kMisc = kBar + 8 * kNumBars;        // tmem base, abort flag
    static constexpr uint32_t kBytes = kMisc + 16;
    static constexpr uint32_t kAlloc = kBytes + 1024;             // slack for 1 KB alignment
    static_assert(kAlloc <= 227 * 1024, "shared memory budget");
    // TMEM columns
    __host__ __device__ static constexpr uint32_t tS(int i) { return i ? 128u : 0u; }
    __host__ __device__ static constexpr uint32_t tO(int i) { return i ? 384u : 256u; }
    static constexpr uint32_t tP = 64;                             // offset of P inside S
};

struct Ctl {
    uint32_t bar0;           // smem address of barrier 0
    volatile int* abort;
    int* err;
    __device__ uint32_t bar(int i) const { return bar0 + 8u * (uint32_t)i; }
    // Waiting threads are suspended (not spinning) until the phase completes,
    // leaving the issue slots to the softmax warps that share their
    // sub-partition; the MMA thread, whose waits for P and for K/V tiles sit
    // on every key tile's critical path, polls instead (spin), which wakes
    // it sooner.
    __device__ bool wait(int i, uint32_t parity, bool spin = false) const {
        auto poll = [&]() {
            return spin ? ptx::mbar_try_wait(bar(i), parity) : ptx::mbar_try_wait_sleep(bar(i), parity);
        };
        if (poll()) return true;
        const long long t0 = clock64();
        for (;;) {
            if (poll()) return true;
            if (*abort) return false;
            if (clock64() - t0 > kWaitLimit) {
                *abort = 1;
                raise_error(err, JANO_ETIMEOUT);
                return false;
            }
        }
    }
    // Warp-uniform wait: lane 0 polls, the verdict is broadcast, so the
    // .sync.aligned tcgen05 operations that follow never run divergently.
    __device__ bool warp_wait(int i, uint32_t parity) const {
        int ok = 0;
        if ((threadIdx.x & 31) == 0) ok = wait(i, parity) ? 1 : 0;
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        return ok != 0;
    }
};

// Row max of 64 values (8 independent chains of 3-input max); with kMask,
// keys >= valid (the ragged last key tile) are left out.
template <bool kMask>
__device__ __forceinline__ float max64(const uint32_t (&s)[64], int valid) {
    float m[8];
#pragma unroll
    for (int a = 0; a < 8; ++a) m[a] = -INFINITY;
#pragma unroll
    for (int e = 0; e < 64; e += 2) {
        float x = __uint_as_float(s[e]), y = __uint_as_float(s[e + 1]);
        if (kMask && e >= valid) x = -INFINITY;
        if (kMask && e + 1 >= valid) y = -INFINITY;
        m[(e >> 1) & 7] = ptx::fmax3(m[(e >> 1) & 7], x, y);
    }
    return fmaxf(ptx::fmax3(m[0], m[1], m[2]), ptx::fmax3(m[3], m[4], fmaxf(m[5], fmaxf(m[6], m[7]))));
}

// 2^x for two lanes on the FMA/ALU pipes, to take part of the exponentials
// off the MUFU unit (which alone would need about as many cycles per key
// tile as the tensor core).  Range reduction x = j + f with j = rint(x)
// (added to the exponent bits) and f in [-1/2, 1/2]; 2^f by a cubic whose
// coefficients were fitted here by Remez exchange for the smallest maximum
// relative error on [-1/2, 1/2]: 7.5e-5 (2^-13.7) in fp32 Horner form, far
// below the 2^-8 rounding of the BF16 P it feeds.  Inputs below -125 are
// clamped so 2^j stays a normal float (such terms are < 2^-125 of the row
// maximum).
__device__ __forceinline__ void exp2_poly2(uint64_t x2, float& ya, float& yb) {
    constexpr float kC0 = 0x1.fff692p-1f, kC1 = 0x1.62f31ap-1f;
    constexpr float kC2 = 0x1.f0de1ap-3f, kC3 = 0x1.c3f76p-5f;
    constexpr float kRound = 12582912.0f;            // 1.5 * 2^23
    float xa, xb;
    ptx::f2split(x2, xa, xb);
    x2 = ptx::f2(fmaxf(xa, -125.0f), fmaxf(xb, -125.0f));
    const uint64_t r2 = ptx::fadd2(x2, ptx::f2(kRound, kRound));     // low bits hold rint(x)
    const uint64_t t2 = ptx::fadd2(r2, ptx::f2(-kRound, -kRound));
    const uint64_t f2 = ptx::ffma2(t2, ptx::f2(-1.f, -1.f), x2);      // f = x - rint(x)
    uint64_t p2 = ptx::ffma2(ptx::f2(kC3, kC3), f2, ptx::f2(kC2, kC2));
    p2 = ptx::ffma2(p2, f2, ptx::f2(kC1, kC1));
    p2 = ptx::ffma2(p2, f2, ptx::f2(kC0, kC0));
    float ra, rb, pa, pb;
    ptx::f2split(r2, ra, rb);
    ptx::f2split(p2, pa, pb);
    const int ja = __float_as_int(ra) - __float_as_int(kRound);
    const int jb = __float_as_int(rb) - __float_as_int(kRound);
    ya = __int_as_float(__float_as_int(pa) + (ja << 23));
    yb = __int_as_float(__float_as_int(pb) + (jb << 23));
}

// Share of the exponentials computed by exp2_poly2, in eighths: pairs whose
// index modulo 8 is below this count (0 = all on MUFU, 1 = an eighth).
#ifndef JANO_EXP2_POLY_EIGHTHS
#define JANO_EXP2_POLY_EIGHTHS 1
#endif

// p = 2^(s*c - m) for 64 values, packed to 32 BF16x2 words; returns sum(p).
template <bool kMask>
__device__ __forceinline__ float exp64(const uint32_t (&s)[64], int valid, float c, float m,
                                       uint32_t* pk) {
    const uint64_t c2 = ptx::f2(c, c), nm2 = ptx::f2(-m, -m);
    uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
    for (int e = 0; e < 64; e += 2) {
        const uint64_t x2 = ptx::ffma2(ptx::f2(__uint_as_float(s[e]), __uint_as_float(s[e + 1])), c2, nm2);
        float a, b;
        if (((e >> 1) & 7) < JANO_EXP2_POLY_EIGHTHS) {
            exp2_poly2(x2, a, b);
        } else {
            float xa, xb;
            ptx::f2split(x2, xa, xb);
            a = ptx::ex2(xa);
            b = ptx::ex2(xb);
        }
        if (kMask && e >= valid) a = 0.f;
        if (kMask && e + 1 >= valid) b = 0.f;
        acc[(e >> 1) & 3] = ptx::fadd2(acc[(e >> 1) & 3], ptx::f2(a, b));
        pk[e >> 1] = ptx::pack_bf16(a, b);
    }
    const uint64_t t = ptx::fadd2(ptx::fadd2(acc[0], acc[1]), ptx::fadd2(acc[2], acc[3]));
    float lo, hi;
    ptx::f2split(t, lo, hi);
    return lo + hi;
}

// One key tile of one query row: the row's 128 S values from TMEM in one
// round trip, row max, lazy O rescale, P = 2^(S*c - m) as BF16 into the upper
// half of the row's S columns.  Warp-uniform control flow throughout.
// kRemote: bar_half is a shared::cluster address (the pair form's barriers
// live in the even CTA) and is arrived on at cluster scope.
template <int HD, bool kMask, bool kRemote = false>
__device__ __forceinline__ void softmax_tile(uint32_t tS, uint32_t tO, uint32_t tP, int j, int valid,
                                             float c, float& m, float& l, uint32_t bar_half) {
    uint32_t s[128];
    ptx::tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
    ptx::tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
    ptx::tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&s[64]));
    ptx::tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&s[96]));
    ptx::tmem_wait_ld();
    const uint32_t(&lo)[64] = *reinterpret_cast<const uint32_t(*)[64]>(&s[0]);
    const uint32_t(&hi)[64] = *reinterpret_cast<const uint32_t(*)[64]>(&s[64]);
    const float mx = fmaxf(max64<kMask>(lo, valid), max64<kMask>(hi, valid - 64));
    const float mxs = mx * c;
    // lazy rescale, decided per warp so the TMEM accesses stay warp-wide:
    // lanes whose max did not grow past 2^8 keep their max (alpha = 1).
    const bool want = mxs > m + 8.0f;
    if (__any_sync(0xFFFFFFFFu, want)) {
        const float m_new = want ? mxs : m;
        if (j > 0) {
            const float alpha = ptx::ex2(m - m_new);
            l *= alpha;
#pragma unroll
            for (int q = 0; q < HD / 32; ++q) {
                uint32_t o[32];
                ptx::tmem_ld32(tO + 32 * q, o);
                ptx::tmem_wait_ld();
                const uint64_t a2 = ptx::f2(alpha, alpha);
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    float lo2, hi2;
                    ptx::f2split(ptx::fmul2(ptx::f2(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), a2), lo2, hi2);
                    o[e] = __float_as_uint(lo2);
                    o[e + 1] = __float_as_uint(hi2);
                }
                ptx::tmem_st32(tO + 32 * q, o);
            }
            ptx::tmem_wait_st();
        }
        m = m_new;
    }
    // upper key half first: its P goes to P columns [32,64) and is handed to
    // the MMA thread, whose P.V runs while the lower half is exponentiated
    uint32_t pk[32];
    l += exp64<kMask>(hi, valid - 64, c, m, pk);
    ptx::tmem_st32(tP + 32, *reinterpret_cast<uint32_t(*)[32]>(pk));
    ptx::tmem_wait_st();
    ptx::tc_fence_before();
    __syncwarp();
    if ((threadIdx.x & 31) == 0) {
        if constexpr (kRemote) ptx::mbar_arrive_cluster(bar_half);
        else ptx::mbar_arrive(bar_half);
    }
    l += exp64<kMask>(lo, valid, c, m, pk);
    ptx::tmem_st32(tP, *reinterpret_cast<uint32_t(*)[32]>(pk));
    ptx::tmem_wait_st();
}

// kSplit: the key-split form (grid z = splits, partials to part_o / part_ml);
// otherwise one CTA takes all keys and writes the normalised BF16 rows.
template <int HD, bool kSplit>
__global__ void __launch_bounds__(kThreads, 1)
attention_kernel(const __grid_constant__ CUtensorMap tmQ,
                 const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV,
                 const int32_t* __restrict__ idx, int n_act, int n_tokens, int heads,
                 float scale_log2, __nv_bfloat16* __restrict__ out, float* __restrict__ part_o,
                 float2* __restrict__ part_ml, int* err) {
    using L = Layout<HD>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = ptx::smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int head = blockIdx.y;
    const int q0 = blockIdx.x * 2 * BM;                // first query row of tile 0
    // key split: CTA z of n_split takes key tiles [kt0, kt1) of the nt_all
    const int nt_all = (n_tokens + BN - 1) / BN;
    const int n_split = kSplit ? (int)gridDim.z : 1, split = kSplit ? (int)blockIdx.z : 0;
    const int kt0 = kSplit ? (int)((long long)nt_all * split / n_split) : 0;
    const int kt1 = kSplit ? (int)((long long)nt_all * (split + 1) / n_split) : nt_all;
    const int nt = kt1 - kt0;                          // key tiles of this CTA

    Ctl ctl;
    ctl.bar0 = base + L::kBar;
    ctl.abort = reinterpret_cast<volatile int*>(gbase + L::kMisc + 4);
    ctl.err = err;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + L::kMisc);

    if (threadIdx.x == 0) {
        ptx::prefetch_tmap(&tmQ);
        ptx::prefetch_tmap(&tmK);
        ptx::prefetch_tmap(&tmV);
        ptx::mbar_init(ctl.bar(L::bQFull), 1);
        for (int s = 0; s < kSlots; ++s) {
            ptx::mbar_init(ctl.bar(L::bFull + s), 1);
            ptx::mbar_init(ctl.bar(L::bEmpty + s), 1);
        }
        for (int s = 0; s < 2; ++s) {
            ptx::mbar_init(ctl.bar(L::bSFull + s), 1);
            ptx::mbar_init(ctl.bar(L::bPFull + s), 4);
            ptx::mbar_init(ctl.bar(L::bPHalf + s), 4);
            ptx::mbar_init(ctl.bar(L::bOFull + s), 1);
        }
        ptx::mbar_init(ctl.bar(L::bFinal), 1);
        *ctl.abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 9) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), 512);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp >= 8) {
      ptx::setmaxnreg_dec<kRegsIssue>();
      if (warp == 8) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int last[kSlots];
            for (int s = 0; s < kSlots; ++s) last[s] = -1;
            ptx::mbar_arrive_expect_tx(ctl.bar(L::bQFull), 2 * L::kTile);
            for (int p = 0; p < L::kPanels; ++p) {
                ptx::tma_load_3d(base + L::kQ0 + p * kPanel, &tmQ, ctl.bar(L::bQFull), p * 64, head, q0);
                ptx::tma_load_3d(base + L::kQ1 + p * kPanel, &tmQ, ctl.bar(L::bQFull), p * 64, head, q0 + BM);
            }
            // load sequence: K_0 V_0 K_1 V_1 ...; load n goes to slot n % kSlots
            for (int n = 0; n < 2 * nt; ++n) {
                const int s = n % kSlots;
                if (!ctl.wait(L::bEmpty + s, ((n / kSlots) & 1) ^ 1)) break;
#ifdef JANO_INJECT_DROP_LOAD
                // failure-path test builds only: this copy is never issued, so
                // the MMA's bounded wait for it runs out (JANO_ETIMEOUT)
                if (n == JANO_INJECT_DROP_LOAD) continue;
#endif
                ptx::mbar_arrive_expect_tx(ctl.bar(L::bFull + s), L::kTile);
                const CUtensorMap* tm = (n & 1) ? &tmV : &tmK;
                for (int p = 0; p < L::kPanels; ++p)
                    ptx::tma_load_3d(base + L::kRing + s * L::kTile + p * kPanel, tm,
                                     ctl.bar(L::bFull + s), p * 64, head, (kt0 + (n >> 1)) * BN);
                last[s] = n;
            }
            // drain: every copy this CTA issued lands before its smem is released
            ptx::mbar_wait(ctl.bar(L::bQFull), 0, kWaitLimit);
            for (int s = 0; s < kSlots; ++s)
                if (last[s] >= 0) ptx::mbar_wait(ctl.bar(L::bFull + s), (last[s] / kSlots) & 1, kWaitLimit);
        }
    } else if (warp == 9) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = ptx::idesc_bf16(BM, BN, false, false);
            constexpr uint32_t idesc_pv = ptx::idesc_bf16(BM, HD, false, true);
            auto slot_of = [](int n) { return n % kSlots; };
            auto wait_full = [&](int n) { return ctl.wait(L::bFull + slot_of(n), (n / kSlots) & 1, true); };
            auto qk = [&](int i, int n) {          // S_i = Q_i K^T, K in load n's slot
                const uint32_t kb = base + L::kRing + slot_of(n) * L::kTile;
                const uint32_t qb = base + (i ? L::kQ1 : L::kQ0);
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kPanel + (kk & 3) * 32;
                    ptx::mma_ss(tmem + L::tS(i), ptx::smem_desc_sw128(qb + off, 16, 1024),
                                ptx::smem_desc_sw128(kb + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
                }
            };
            // O_i += P_i V over key sixteenths [k0, k1); V in load n's slot
            auto pv = [&](int i, int n, int k0, int k1, bool acc) {
                const uint32_t vb = base + L::kRing + slot_of(n) * L::kTile;
#pragma unroll
                for (int kk = k0; kk < k1; ++kk)
                    ptx::mma_ts(tmem + L::tO(i), tmem + L::tS(i) + L::tP + kk * 8,
                                ptx::smem_desc_sw128(vb + kk * 2048, kPanel, 1024), idesc_pv,
                                (acc || kk > k0) ? 1u : 0u);
            };
            // P_i of tile j: upper key half as soon as it is published, then the lower half
            auto pv_tile = [&](int i, int n, int j) -> bool {
                if (!ctl.wait(L::bPHalf + i, j & 1, true)) return false;
                ptx::tc_fence_after();
                pv(i, n, BN / 32, BN / 16, j > 0);
                if (!ctl.wait(L::bPFull + i, j & 1, true)) return false;
                ptx::tc_fence_after();
                pv(i, n, 0, BN / 32, true);
                return true;
            };
            bool ok = ctl.wait(L::bQFull, 0) && wait_full(0);
            if (ok) {
                ptx::tc_fence_after();
                qk(0, 0);
                ptx::mma_commit(ctl.bar(L::bSFull + 0));
                qk(1, 0);
                ptx::mma_commit(ctl.bar(L::bSFull + 1));
                ptx::mma_commit(ctl.bar(L::bEmpty + slot_of(0)));
            }
            for (int j = 1; ok && j < nt; ++j) {
                const int nk = 2 * j, nv = 2 * j - 1;        // loads of K_j and V_{j-1}
                if (!wait_full(nv) || !wait_full(nk)) { ok = false; break; }
                if (!pv_tile(0, nv, j - 1)) { ok = false; break; }
                qk(0, nk);
                ptx::mma_commit(ctl.bar(L::bSFull + 0));
                if (!pv_tile(1, nv, j - 1)) { ok = false; break; }
                ptx::mma_commit(ctl.bar(L::bEmpty + slot_of(nv)));
                qk(1, nk);
                ptx::mma_commit(ctl.bar(L::bSFull + 1));
                ptx::mma_commit(ctl.bar(L::bEmpty + slot_of(nk)));
            }
            if (ok) {
                const int nv = 2 * nt - 1;
                ok = wait_full(nv) && pv_tile(0, nv, nt - 1);
                if (ok) {
                    ptx::mma_commit(ctl.bar(L::bOFull + 0));
                    ok = pv_tile(1, nv, nt - 1);
                }
                if (ok) {
                    ptx::mma_commit(ctl.bar(L::bOFull + 1));
                    ptx::mma_commit(ctl.bar(L::bEmpty + slot_of(nv)));
                }
            }
            // all MMAs of this CTA complete before TMEM can be released
            ptx::mma_commit(ctl.bar(L::bFinal));
            ptx::mbar_wait(ctl.bar(L::bFinal), 0, kWaitLimit);
        }
      }
    } else {
        ptx::setmaxnreg_inc<kRegsSoftmax>();
        // ------------------------------------------------------------ softmax WG i
        const int i = warp >> 2;                      // query tile of this warpgroup
        const int q = warp & 3;                       // TMEM lane quarter of this warp
        const int row = q * 32 + lane;
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        const uint32_t tS = tmem + lane_off + L::tS(i);
        const uint32_t tO = tmem + lane_off + L::tO(i);
        const int qi = q0 + i * BM + row;
        int t_out = -1;
        if (qi < n_act) {
            // idx contract: in range and strictly ascending; a row that breaks
            // it is reported and not written
            t_out = __ldg(idx + qi);
            if (t_out < 0 || t_out >= n_tokens || (qi > 0 && __ldg(idx + qi - 1) >= t_out)) {
                raise_error(err, JANO_EINDEX);
                t_out = -1;
            }
        }
        float m = -INFINITY, l = 0.f;
        // valid keys in this CTA's last tile (only the sequence's last tile is ragged)
        const int tail = kt1 == nt_all ? n_tokens - (nt_all - 1) * BN : BN;
        bool ok = true;
        for (int j = 0; j < nt; ++j) {
            if (!ctl.warp_wait(L::bSFull + i, j & 1)) { ok = false; break; }
            ptx::tc_fence_after();
            if (j < nt - 1 || tail == BN)
                softmax_tile<HD, false>(tS, tO, tS + L::tP, j, BN, scale_log2, m, l, ctl.bar(L::bPHalf + i));
            else
                softmax_tile<HD, true>(tS, tO, tS + L::tP, j, tail, scale_log2, m, l, ctl.bar(L::bPHalf + i));
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(ctl.bar(L::bPFull + i));
        }
        // ------------------------------------------------------------ epilogue
        const bool done = ok && ctl.warp_wait(L::bOFull + i, 0);
        if constexpr (kSplit) {
            // a CTA that gave up leaves a marker (l < 0, impossible for a sum of
            // exponentials) instead of its partial, so the merge skips the row
            if (!done && qi < n_act)
                part_ml[((size_t)split * n_act + qi) * heads + head] = make_float2(-INFINITY, -1.0f);
        }
        if (done) {
            ptx::tc_fence_after();
            if constexpr (!kSplit) {
                const float inv = 1.0f / l;
                __nv_bfloat16* orow = out + ((size_t)(t_out < 0 ? 0 : t_out) * heads + head) * HD;
#pragma unroll
                for (int c = 0; c < HD / 32; ++c) {
                    uint32_t o[32];
                    ptx::tmem_ld32(tO + 32 * c, o);
                    ptx::tmem_wait_ld();
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        pk[e] = ptx::pack_bf16(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
                    if (t_out >= 0) {
                        // streaming stores: the output rows are not read again here,
                        // so they should leave L2 early rather than linger dirty
                        uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
                        for (int v = 0; v < 4; ++v)
                            __stcs(dst + v, make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]));
                    }
                }
            } else {
                // key split: this CTA's unnormalised O (fp32) with its row max m
                // (log2 domain) and sum l, for the combine pass
                const bool live = qi < n_act;
                const size_t prow = ((size_t)split * n_act + (live ? qi : 0)) * heads + head;
                float4* po = reinterpret_cast<float4*>(part_o + prow * HD);
#pragma unroll
                for (int c = 0; c < HD / 32; ++c) {
                    uint32_t o[32];
                    ptx::tmem_ld32(tO + 32 * c, o);
                    ptx::tmem_wait_ld();
                    if (live) {
#pragma unroll
                        for (int v = 0; v < 8; ++v)
                            po[8 * c + v] = make_float4(__uint_as_float(o[4 * v]), __uint_as_float(o[4 * v + 1]),
                                                        __uint_as_float(o[4 * v + 2]), __uint_as_float(o[4 * v + 3]));
                    }
                }
                if (live) part_ml[prow] = make_float2(m, l);
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 9) ptx::tmem_dealloc(tmem, 512);
}

// Merge of the key-split partials: one warp per (query, head) row; lane
// holds HD/32 consecutive columns.  With M = max_s m_s and w_s = 2^(m_s - M),
//   out[idx[i], h] = sum_s w_s O_s / sum_s w_s l_s,
// summed over the splits in order (deterministic).  Rows with a missing
// partial (a timed-out range) or a bad index are left untouched.
template <int HD>
__global__ void __launch_bounds__(256)
attention_combine_kernel(const float* __restrict__ part_o, const float2* __restrict__ part_ml,
                         const int32_t* __restrict__ idx, int n_act, int n_tokens, int heads,
                         int n_split, __nv_bfloat16* __restrict__ out, int* err) {
    constexpr int E = HD / 32;
    const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    const long long rows = (long long)n_act * heads;
    if (row >= rows) return;
    const int qi = (int)(row / heads), head = (int)(row % heads);
    const int t = __ldg(idx + qi);
    if (t < 0 || t >= n_tokens || (qi > 0 && __ldg(idx + qi - 1) >= t)) {
        if (lane == 0) raise_error(err, JANO_EINDEX);
        return;
    }
    float M = -INFINITY;
    bool missing = false;
    for (int z = 0; z < n_split; ++z) {
        const float2 ml = part_ml[z * rows + row];
        missing |= ml.y < 0.0f;
        M = fmaxf(M, ml.x);
    }
    // a key range whose CTA timed out (JANO_ETIMEOUT already raised) left no
    // partial: the row is not written, as in the unsplit kernel
    if (missing) return;
    float acc[E], L = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
    for (int z = 0; z < n_split; ++z) {
        const float2 ml = part_ml[z * rows + row];
        const float w = ptx::ex2(ml.x - M);
        L = fmaf(w, ml.y, L);
        const float* src = part_o + (z * rows + row) * HD + lane * E;
        float v[E];
        if constexpr (E == 4) {
            const float4 x = *reinterpret_cast<const float4*>(src);
            v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
        } else {
            const float2 x = *reinterpret_cast<const float2*>(src);
            v[0] = x.x; v[1] = x.y;
        }
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = fmaf(w, v[e], acc[e]);
    }
    const float inv = 1.0f / L;
    __nv_bfloat16* dst = out + ((size_t)t * heads + head) * HD + lane * E;
    if constexpr (E == 4) {
        *reinterpret_cast<uint2*>(dst) = make_uint2(ptx::pack_bf16(acc[0] * inv, acc[1] * inv),
                                                    ptx::pack_bf16(acc[2] * inv, acc[3] * inv));
    } else {
        *reinterpret_cast<uint32_t*>(dst) = ptx::pack_bf16(acc[0] * inv, acc[1] * inv);
    }
}

// ---------------------------------------------------------------------------
// CTA-pair form (d = 128, keys not split).  A cluster of two CTAs on two SMs
// takes four 128-query tiles of one head, two per CTA as above, and runs the
// MMAs of both CTAs as pair MMAs (M = 256: query rows 0-127 from the even
// CTA's shared memory and tensor memory, 128-255 from the odd CTA's), issued
// by one thread of the even CTA.  The B operand of a pair MMA is split by N
// between the two CTAs, so each CTA stages only half of every key tile: for
// S = Q K^T keys [64 r, 64 r + 64) of the tile (all 128 columns), for
// O += P V columns [64 r, 64 r + 64) of V (all 128 keys), r = the CTA's rank.
// Per key tile an SM therefore receives 32 KB instead of 64 KB, and its
// shared-memory port moves about 160 KB instead of 256 KB.  Every load is a
// plain TMA load into the loading CTA's own shared memory (no multicast).
//
// Hand-offs between the two CTAs:
//   - each CTA's copies complete on its own "landed" barriers; a relay thread
//     of each CTA then arrives (cluster scope) on the even CTA's "full"
//     barrier (2 arrivals: one per CTA), which the MMA thread waits on;
//   - softmax warps of both CTAs publish P on the even CTA's P barriers
//     (8 warp arrivals);
//   - the MMA thread's commits are multicast to both CTAs (S ready, O ready,
//     ring slot free, all MMAs done);
//   - a CTA that gives up on a wait sets its own abort flag and the peer's;
//   - tensor memory is allocated and freed at the same columns in both CTAs,
//     and a cluster barrier ends the kernel, so neither CTA leaves while the
//     pair's MMAs or the peer's remote arrivals may still touch it.
// Every mbarrier wait is bounded.
constexpr int kPairSlots = 8;                 // ring of K/V half tiles
constexpr uint32_t kHalfTile = 16384;         // one K or V half tile (BF16)
constexpr uint32_t kHalfPanel = 8192;         // 64 rows x 128 bytes

struct PairLayout {
    static constexpr uint32_t kQ0 = 0;
    static constexpr uint32_t kQ1 = 2 * kPanel;
    static constexpr uint32_t kRing = 4 * kPanel;
    static constexpr uint32_t kBar = kRing + kPairSlots * kHalfTile;
    static constexpr int bQLand = 0;                        // own Q tiles landed (tx)
    static constexpr int bQFull = 1;                        // even CTA: both relays
    static constexpr int bLand = 2;                         // [kPairSlots] own half landed (tx)
    static constexpr int bFull = bLand + kPairSlots;        // [kPairSlots] even CTA: both relays
    static constexpr int bEmpty = bFull + kPairSlots;       // [kPairSlots] commit, both CTAs
    static constexpr int bSFull = bEmpty + kPairSlots;      // [2]
    static constexpr int bPFull = bSFull + 2;               // [2] even CTA: 8 warp arrivals
    static constexpr int bPHalf = bPFull + 2;               // [2] even CTA: 8 warp arrivals
    static constexpr int bOFull = bPHalf + 2;               // [2]
    static constexpr int bFinal = bOFull + 2;
    static constexpr int kNumBars = bFinal + 1;
    static constexpr uint32_t kMisc = kBar + 8 * kNumBars;  // tmem base, abort flag
    static constexpr uint32_t kBytes = kMisc + 16;
    static constexpr uint32_t kAlloc = kBytes + 1024;
    static_assert(kAlloc <= 227 * 1024, "shared memory budget");
};

struct PairCtl {
    uint32_t bar0;           // local address of barrier 0
    uint32_t lead_bar0;      // shared::cluster address of barrier 0 in the even CTA
    uint32_t peer_abort;     // shared::cluster address of the peer's abort flag
    volatile int* abort;
    int* err;
    __device__ uint32_t bar(int i) const { return bar0 + 8u * (uint32_t)i; }
    __device__ uint32_t lead(int i) const { return lead_bar0 + 8u * (uint32_t)i; }
    __device__ void give_up() const {
        *abort = 1;
        ptx::st_cluster_u32(peer_abort, 1u);
        raise_error(err, JANO_ETIMEOUT);
    }
    // Bounded wait; stops early once either CTA of the pair has given up.
    // cluster: acquire at cluster scope, for the barriers that other CTAs'
    // threads arrive on (the even CTA's full and P barriers); the others only
    // receive this CTA's arrivals, its copies and tensor-core commits.
    __device__ bool wait(int i, uint32_t parity, bool spin = false, bool cluster = false) const {
        auto poll = [&]() {
            if (cluster)
                return spin ? ptx::mbar_try_wait_cluster(bar(i), parity)
                            : ptx::mbar_try_wait_cluster_sleep(bar(i), parity);
            return spin ? ptx::mbar_try_wait(bar(i), parity) : ptx::mbar_try_wait_sleep(bar(i), parity);
        };
        if (poll()) return true;
        const long long t0 = clock64();
        for (;;) {
            if (poll()) return true;
            if (*abort) return false;
            if (clock64() - t0 > kWaitLimit) {
                give_up();
                return false;
            }
        }
    }
    __device__ bool warp_wait(int i, uint32_t parity) const {
        int ok = 0;
        if ((threadIdx.x & 31) == 0) ok = wait(i, parity) ? 1 : 0;
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        return ok != 0;
    }
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
attention_pair_kernel(const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV,
                      const int32_t* __restrict__ idx, int n_act, int n_tokens, int heads,
                      float scale_log2, __nv_bfloat16* __restrict__ out, int* err) {
    constexpr int HD = 128;
    using L = PairLayout;
    using LS = Layout<HD>;                      // TMEM columns as in the single-CTA form
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = ptx::smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = ptx::cluster_ctarank();
    const bool lead = rank == 0;
    const int head = blockIdx.y;
    const int q0 = ((int)(blockIdx.x >> 1) * 4 + 2 * (int)rank) * BM;   // this CTA's tile 0
    const int nt = (n_tokens + BN - 1) / BN;

    PairCtl ctl;
    ctl.bar0 = base + L::kBar;
    ctl.lead_bar0 = ptx::mapa_shared(ctl.bar0, 0);
    ctl.abort = reinterpret_cast<volatile int*>(gbase + L::kMisc + 4);
    ctl.peer_abort = ptx::mapa_shared(base + L::kMisc + 4, rank ^ 1u);
    ctl.err = err;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + L::kMisc);

    if (threadIdx.x == 0) {
        ptx::prefetch_tmap(&tmQ);
        ptx::prefetch_tmap(&tmK);
        ptx::prefetch_tmap(&tmV);
        ptx::mbar_init(ctl.bar(L::bQLand), 1);
        ptx::mbar_init(ctl.bar(L::bQFull), 2);
        for (int s = 0; s < kPairSlots; ++s) {
            ptx::mbar_init(ctl.bar(L::bLand + s), 1);
            ptx::mbar_init(ctl.bar(L::bFull + s), 2);
            ptx::mbar_init(ctl.bar(L::bEmpty + s), 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(ctl.bar(L::bSFull + i), 1);
            ptx::mbar_init(ctl.bar(L::bPFull + i), 8);
            ptx::mbar_init(ctl.bar(L::bPHalf + i), 8);
            ptx::mbar_init(ctl.bar(L::bOFull + i), 1);
        }
        ptx::mbar_init(ctl.bar(L::bFinal), 1);
        *ctl.abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 9) {
        ptx::tmem_alloc_pair(ptx::smem_u32(tmem_slot), 512);
        ptx::tmem_relinquish_pair();
    }
    // both CTAs' barriers initialised and tensor memory allocated before any
    // cross-CTA arrival or pair MMA
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync_all();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp >= 8) {
      ptx::setmaxnreg_dec<kRegsIssue>();
      if (warp == 8) {
        // ------------------------------------------------------------ producer (each CTA)
        if (lane == 0) {
            int last[kPairSlots];
            for (int s = 0; s < kPairSlots; ++s) last[s] = -1;
            ptx::mbar_arrive_expect_tx(ctl.bar(L::bQLand), 4 * kPanel);
            for (int p = 0; p < 2; ++p) {
                ptx::tma_load_3d(base + L::kQ0 + p * kPanel, &tmQ, ctl.bar(L::bQLand), p * 64, head, q0);
                ptx::tma_load_3d(base + L::kQ1 + p * kPanel, &tmQ, ctl.bar(L::bQLand), p * 64, head, q0 + BM);
            }
            // load n: K half (n even) or V half (n odd) of key tile n/2, into slot n % kPairSlots
            for (int n = 0; n < 2 * nt; ++n) {
                const int s = n % kPairSlots;
                if (!ctl.wait(L::bEmpty + s, ((n / kPairSlots) & 1) ^ 1)) break;
#ifdef JANO_INJECT_DROP_LOAD
                if (n == JANO_INJECT_DROP_LOAD) continue;    // failure-path test builds only
#endif
                const uint32_t dst = base + L::kRing + s * kHalfTile;
                const int kt = n >> 1;
                ptx::mbar_arrive_expect_tx(ctl.bar(L::bLand + s), kHalfTile);
                if ((n & 1) == 0) {
                    // keys [64 r, 64 r + 64) of the tile, columns 0-63 and 64-127
                    const int k0 = kt * BN + 64 * (int)rank;
                    ptx::tma_load_3d(dst, &tmK, ctl.bar(L::bLand + s), 0, head, k0);
                    ptx::tma_load_3d(dst + kHalfPanel, &tmK, ctl.bar(L::bLand + s), 64, head, k0);
                } else {
                    // columns [64 r, 64 r + 64) of V, keys 0-63 and 64-127 of the tile
                    const int c0 = 64 * (int)rank;
                    ptx::tma_load_3d(dst, &tmV, ctl.bar(L::bLand + s), c0, head, kt * BN);
                    ptx::tma_load_3d(dst + kHalfPanel, &tmV, ctl.bar(L::bLand + s), c0, head, kt * BN + 64);
                }
                last[s] = n;
            }
            // drain: every copy this CTA issued lands before its smem is released
            ptx::mbar_wait(ctl.bar(L::bQLand), 0, kWaitLimit);
            for (int s = 0; s < kPairSlots; ++s)
                if (last[s] >= 0) ptx::mbar_wait(ctl.bar(L::bLand + s), (last[s] / kPairSlots) & 1, kWaitLimit);
        }
      } else if (warp == 10) {
        // ------------------------------------------------------------ relay (each CTA)
        // this CTA's half of a stage has landed -> one arrival on the even CTA's full barrier
        if (lane == 0 && ctl.wait(L::bQLand, 0)) {
            ptx::mbar_arrive_cluster(ctl.lead(L::bQFull));
            for (int n = 0; n < 2 * nt; ++n) {
                const int s = n % kPairSlots;
                if (!ctl.wait(L::bLand + s, (n / kPairSlots) & 1, true)) break;
                ptx::mbar_arrive_cluster(ctl.lead(L::bFull + s));
            }
        }
      } else if (warp == 9 && lead) {
        // ------------------------------------------------------------ MMA issuer (even CTA)
        if (lane == 0) {
            constexpr uint32_t idesc_qk = ptx::idesc_bf16(2 * BM, BN, false, false);
            constexpr uint32_t idesc_pv = ptx::idesc_bf16(2 * BM, HD, false, true);
            constexpr uint16_t kBoth = 0x3;
            auto slot_of = [](int n) { return n % kPairSlots; };
            auto wait_full = [&](int n) { return ctl.wait(L::bFull + slot_of(n), (n / kPairSlots) & 1, true, true); };
            auto commit = [&](int b) { ptx::mma_commit_pair_mc(ctl.bar(b), kBoth); };
            auto qk = [&](int i, int n) {          // S_i = Q_i K^T, K halves in load n's slot
                const uint32_t kb = base + L::kRing + slot_of(n) * kHalfTile;
                const uint32_t qb = base + (i ? L::kQ1 : L::kQ0);
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    ptx::mma_ss_pair(tmem + LS::tS(i),
                                     ptx::smem_desc_sw128(qb + (kk >> 2) * kPanel + (kk & 3) * 32, 16, 1024),
                                     ptx::smem_desc_sw128(kb + (kk >> 2) * kHalfPanel + (kk & 3) * 32, 16, 1024),
                                     idesc_qk, kk > 0 ? 1u : 0u);
                }
            };
            // O_i += P_i V over key sixteenths [k0, k1); V halves in load n's slot
            auto pv = [&](int i, int n, int k0, int k1, bool acc) {
                const uint32_t vb = base + L::kRing + slot_of(n) * kHalfTile;
#pragma unroll
                for (int kk = k0; kk < k1; ++kk)
                    ptx::mma_ts_pair(tmem + LS::tO(i), tmem + LS::tS(i) + LS::tP + kk * 8,
                                     ptx::smem_desc_sw128(vb + kk * 2048, kHalfTile, 1024), idesc_pv,
                                     (acc || kk > k0) ? 1u : 0u);
            };
            auto pv_tile = [&](int i, int n, int j) -> bool {
                if (!ctl.wait(L::bPHalf + i, j & 1, true, true)) return false;
                ptx::tc_fence_after();
                pv(i, n, BN / 32, BN / 16, j > 0);
                if (!ctl.wait(L::bPFull + i, j & 1, true, true)) return false;
                ptx::tc_fence_after();
                pv(i, n, 0, BN / 32, true);
                return true;
            };
            bool ok = ctl.wait(L::bQFull, 0, false, true) && wait_full(0);
            if (ok) {
                ptx::tc_fence_after();
                qk(0, 0);
                commit(L::bSFull + 0);
                qk(1, 0);
                commit(L::bSFull + 1);
                commit(L::bEmpty + slot_of(0));
            }
            for (int j = 1; ok && j < nt; ++j) {
                const int nk = 2 * j, nv = 2 * j - 1;        // loads of K_j and V_{j-1}
                if (!wait_full(nv) || !wait_full(nk)) { ok = false; break; }
                ptx::tc_fence_after();
                if (!pv_tile(0, nv, j - 1)) { ok = false; break; }
                qk(0, nk);
                commit(L::bSFull + 0);
                if (!pv_tile(1, nv, j - 1)) { ok = false; break; }
                commit(L::bEmpty + slot_of(nv));
                qk(1, nk);
                commit(L::bSFull + 1);
                commit(L::bEmpty + slot_of(nk));
            }
            if (ok) {
                const int nv = 2 * nt - 1;
                ok = wait_full(nv);
                if (ok) {
                    ptx::tc_fence_after();
                    ok = pv_tile(0, nv, nt - 1);
                }
                if (ok) {
                    commit(L::bOFull + 0);
                    ok = pv_tile(1, nv, nt - 1);
                }
                if (ok) {
                    commit(L::bOFull + 1);
                    commit(L::bEmpty + slot_of(nv));
                }
            }
            // every pair MMA is complete (in both CTAs) before tensor memory is released
            commit(L::bFinal);
            ptx::mbar_wait(ctl.bar(L::bFinal), 0, kWaitLimit);
        }
      } else if (warp == 9) {
        // odd CTA: the final commit's arrival has landed here before this CTA
        // can leave (the even CTA commits it on every path, aborts included)
        if (lane == 0) ptx::mbar_wait(ctl.bar(L::bFinal), 0, kWaitLimit);
      }
    } else {
        ptx::setmaxnreg_inc<kRegsSoftmax>();
        // ------------------------------------------------------------ softmax WG i (each CTA)
        const int i = warp >> 2;
        const int q = warp & 3;
        const int row = q * 32 + lane;
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        const uint32_t tS = tmem + lane_off + LS::tS(i);
        const uint32_t tO = tmem + lane_off + LS::tO(i);
        const int qi = q0 + i * BM + row;
        int t_out = -1;
        if (qi < n_act) {
            t_out = __ldg(idx + qi);
            if (t_out < 0 || t_out >= n_tokens || (qi > 0 && __ldg(idx + qi - 1) >= t_out)) {
                raise_error(err, JANO_EINDEX);
                t_out = -1;
            }
        }
        float m = -INFINITY, l = 0.f;
        const int tail = n_tokens - (nt - 1) * BN;
        bool ok = true;
        for (int j = 0; j < nt; ++j) {
            if (!ctl.warp_wait(L::bSFull + i, j & 1)) { ok = false; break; }
            ptx::tc_fence_after();
            if (j < nt - 1 || tail == BN)
                softmax_tile<HD, false, true>(tS, tO, tS + LS::tP, j, BN, scale_log2, m, l, ctl.lead(L::bPHalf + i));
            else
                softmax_tile<HD, true, true>(tS, tO, tS + LS::tP, j, tail, scale_log2, m, l, ctl.lead(L::bPHalf + i));
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive_cluster(ctl.lead(L::bPFull + i));
        }
        if (ok && ctl.warp_wait(L::bOFull + i, 0)) {
            ptx::tc_fence_after();
            const float inv = 1.0f / l;
            __nv_bfloat16* orow = out + ((size_t)(t_out < 0 ? 0 : t_out) * heads + head) * HD;
#pragma unroll
            for (int c = 0; c < HD / 32; ++c) {
                uint32_t o[32];
                ptx::tmem_ld32(tO + 32 * c, o);
                ptx::tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    pk[e] = ptx::pack_bf16(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
                if (t_out >= 0) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        __stcs(dst + v, make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]));
                }
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    // neither CTA leaves (or frees its tensor memory) while the pair's MMAs or
    // the peer's remote arrivals may still reach it
    ptx::cluster_sync_all();
    ptx::tc_fence_after();
    if (warp == 9) ptx::tmem_dealloc_pair(tmem, 512);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 3D map over [rows][heads][d] BF16, box = 64 columns x 1 head x box_rows rows.
bool make_map(CUtensorMap* m, const void* ptr, int rows, int heads, int d, int box_rows = 128) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)rows};
    const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)heads * d * 2};
    const cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
    const cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int HD, bool kSplit>
cudaError_t launch_hd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                      const int32_t* idx, int n_act, int n_tokens, int heads, float scale,
                      void* out, int n_split, void* ws, int* err, cudaStream_t st) {
    using L = Layout<HD>;
    // the shared-memory opt-in is per device: remember which devices have it
    static DeviceOnce ready;
    int dev = 0;
    cudaGetDevice(&dev);
    if (!ready.done(dev)) {
        // the register split assumes exactly kRegsLaunch registers per thread
        // at launch; anything else could leave an increase waiting for good
        cudaFuncAttributes fa;
        cudaError_t e = cudaFuncGetAttributes(&fa, attention_kernel<HD, kSplit>);
        if (e != cudaSuccess) return e;
        if (fa.numRegs != kRegsLaunch) return cudaErrorInvalidConfiguration;
        e = cudaFuncSetAttribute(attention_kernel<HD, kSplit>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)L::kAlloc);
        if (e != cudaSuccess) return e;
        ready.mark(dev);
    }
    const int q_tiles = (n_act + BM - 1) / BM;
    const dim3 grid((q_tiles + 1) / 2, heads, n_split);
    const float scale_log2 = scale * 1.4426950408889634f;
    float* part_o = nullptr;
    float2* part_ml = nullptr;
    if (kSplit) {
        part_o = static_cast<float*>(ws);
        part_ml = reinterpret_cast<float2*>(static_cast<char*>(ws) +
                                            attention_partials_bytes(n_act, heads, HD, n_split));
    }
    attention_kernel<HD, kSplit><<<grid, kThreads, L::kAlloc, st>>>(
        mq, mk, mv, idx, n_act, n_tokens, heads, scale_log2,
        static_cast<__nv_bfloat16*>(out), part_o, part_ml, err);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || !kSplit) return e;
    const long long rows = (long long)n_act * heads;
    attention_combine_kernel<HD><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(
        part_o, part_ml, idx, n_act, n_tokens, heads, n_split, static_cast<__nv_bfloat16*>(out), err);
    return cudaGetLastError();
}

// The CTA-pair kernel (d = 128, keys not split): clusters of two CTAs, four
// query tiles per cluster.
cudaError_t launch_pair(const void* q, const void* k, const void* v, const int32_t* idx, int n_act,
                        int n_tokens, int heads, float scale, void* out, int* err, cudaStream_t st) {
    static DeviceOnce ready;
    int dev = 0;
    cudaGetDevice(&dev);
    if (!ready.done(dev)) {
        cudaFuncAttributes fa;
        cudaError_t e = cudaFuncGetAttributes(&fa, attention_pair_kernel);
        if (e != cudaSuccess) return e;
        if (fa.numRegs != kRegsLaunch) return cudaErrorInvalidConfiguration;
        e = cudaFuncSetAttribute(attention_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)PairLayout::kAlloc);
        if (e != cudaSuccess) return e;
        ready.mark(dev);
    }
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, q, n_act, heads, 128, 128) || !make_map(&mk, k, n_tokens, heads, 128, 64) ||
        !make_map(&mv, v, n_tokens, heads, 128, 64))
        return cudaErrorInvalidValue;
    const int q_tiles = (n_act + BM - 1) / BM;
    const dim3 grid(2 * ((q_tiles + 3) / 4), heads, 1);
    attention_pair_kernel<<<grid, kThreads, PairLayout::kAlloc, st>>>(
        mq, mk, mv, idx, n_act, n_tokens, heads, scale * 1.4426950408889634f,
        static_cast<__nv_bfloat16*>(out), err);
    return cudaGetLastError();
}

}  // namespace

size_t attention_partials_bytes(int n_act, int heads, int d, int n_split) {
    const size_t o = (size_t)n_split * n_act * heads * d * sizeof(float);
    return (o + 255) / 256 * 256;
}

size_t attention_workspace_bytes(int n_act, int heads, int d, int n_split) {
    if (n_split <= 1) return 0;
    return attention_partials_bytes(n_act, heads, d, n_split) + (size_t)n_split * n_act * heads * 8;
}

int attention_key_tiles(int n_tokens) { return (n_tokens + BN - 1) / BN; }

// Key split with the shortest modelled time.  z splits give z*C CTAs over S
// SMs (one CTA per SM): floor(w) full rounds, w = z C / S, and for a
// partial last round of fraction f a cost of 0.7 + 0.3 f rounds (a part-full
// round runs faster per CTA, being less contended); each CTA costs its
// nt / z key tiles plus the equivalent of 12 tiles (set-up, pipeline fill
// and drain, its partial rows and their merge).  The two constants were
// fitted to measured sweeps of split counts on B200 (due sets of 1.6K to
// 41.6K queries, 5 to 40 heads, 32.8K and 75.6K keys), where the modelled
// choice lands within 4% of the fastest split.  At least 8 key tiles per CTA.
int attention_split_count(int n_act, int n_tokens, int heads, int sms) {
    if (n_act <= 0 || sms <= 0) return 1;
    const long long ctas = (long long)((n_act + 2 * BM - 1) / (2 * BM)) * heads;
    const int nt = attention_key_tiles(n_tokens);
    int best = 1;
    double best_t = 0.0;
    for (int z = 1; z <= 16 && nt / z >= 8; ++z) {
        const double w = (double)(ctas * z) / sms;
        const double full = std::floor(w), f = w - full;
        const double rounds = full + (f > 1e-9 ? 0.7 + 0.3 * f : 0.0);
        const double t = rounds * ((double)nt / z + 12.0);
        if (z == 1 || t < best_t * (1.0 - 1e-9)) {
            best_t = t;
            best = z;
        }
    }
    return best;
}

cudaError_t launch_active_attention(const void* q, const void* k, const void* v,
                                    const int32_t* idx, int n_act, int n_tokens,
                                    int heads, int d, float scale, void* out,
                                    int* err, cudaStream_t st, int n_split, void* ws) {
    if (n_act <= 0) return cudaSuccess;
#if JANO_ATTN_PAIR
    if (d == 128 && n_split == 1)
        return launch_pair(q, k, v, idx, n_act, n_tokens, heads, scale, out, err, st);
#endif
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, q, n_act, heads, d) || !make_map(&mk, k, n_tokens, heads, d) ||
        !make_map(&mv, v, n_tokens, heads, d))
        return cudaErrorInvalidValue;
    if (n_split < 1 || n_split > attention_key_tiles(n_tokens) || (n_split > 1 && !ws))
        return cudaErrorInvalidValue;
    if (n_split > 1) {
        if (d == 128)
            return launch_hd<128, true>(mq, mk, mv, idx, n_act, n_tokens, heads, scale, out, n_split, ws, err, st);
        return launch_hd<64, true>(mq, mk, mv, idx, n_act, n_tokens, heads, scale, out, n_split, ws, err, st);
    }
    if (d == 128)
        return launch_hd<128, false>(mq, mk, mv, idx, n_act, n_tokens, heads, scale, out, 1, nullptr, err, st);
    return launch_hd<64, false>(mq, mk, mv, idx, n_act, n_tokens, heads, scale, out, 1, nullptr, err, st);
}

}  // namespace jano
