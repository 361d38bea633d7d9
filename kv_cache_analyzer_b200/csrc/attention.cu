// attention.cu -- active-query attention over the whole cached K/V, outputs
// scattered back to their token rows (Jano pages: nl technical summary,
// Methodologie 2 "KV Cache Mechanisme": cached K/V of frozen tokens are
// concatenated with the active queries, no position restoration, attention
// being invariant to the order of keys/values; ko 2.B; pt 2.B).
//
//   out[idx[i], h] = softmax_j(scale * q_act[i,h] . k_cache[j,h]) @ v_cache[:, h]
//
// Flash-style forward on the 5th-generation tensor cores.  One CTA per
// (128-query tile, head); 6 warps:
//   warp 0     TMA producer: Q tile once, then K_j / V_j tiles (128 keys x d)
//              into a 2-stage shared-memory ring (128-byte swizzle, boxes of
//              64 columns), completion counted on mbarriers.
//   warp 1     allocates 512 TMEM columns; one lane issues every tcgen05.mma:
//              S_j = Q K_j^T (both K-major in smem) into TMEM buffer j%2, then
//              O += P_{j-1} V_{j-1} with P read from TMEM (A operand) and V
//              MN-major from smem.  tcgen05.commit arrives on the barriers
//              that free smem stages and hand S to the softmax warps.
//   warps 2-5  softmax: thread = one query row = one TMEM lane.  Reads its S
//              row (128 fp32) with tcgen05.ld, masks the ragged last key tile,
//              keeps the running max in the log2 domain and rescales O in TMEM
//              only when the max grows by more than 2^8 (lazy rescale), writes
//              P as packed BF16 into TMEM, and finally normalises O and stores
//              the BF16 row to out[idx[i]].
// TMEM columns: S0 [0,128) S1 [128,256) O [256,256+d) P0, P1 (64 each).
// Every wait is bounded; on timeout the CTA records JANO_ETIMEOUT, drains its
// own copies and MMAs, frees TMEM and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "jano_common.cuh"

namespace jano {
namespace {

constexpr int BM = 128;            // queries per tile
constexpr int BN = 128;            // keys per tile
constexpr int kStages = 2;
constexpr int kThreads = 192;
constexpr uint32_t kPanel = 128 * 128;   // bytes of one 128-row x 64-col BF16 panel
constexpr long long kWaitLimit = 1ll << 31;  // cycles (~1 s)

template <int HD>
struct Layout {
    static constexpr int kPanels = HD / 64;
    static constexpr uint32_t kTile = kPanels * kPanel;           // Q, K or V tile bytes
    static constexpr uint32_t kQ = 0;
    static constexpr uint32_t kK = kQ + kTile;
    static constexpr uint32_t kV = kK + kStages * kTile;
    static constexpr uint32_t kBar = kV + kStages * kTile;
    // barrier slots
    static constexpr int bQFull = 0;
    static constexpr int bKFull = 1;
    static constexpr int bKEmpty = bKFull + kStages;
    static constexpr int bVFull = bKEmpty + kStages;
    static constexpr int bVEmpty = bVFull + kStages;
    static constexpr int bSFull = bVEmpty + kStages;   // [2]
    static constexpr int bSFree = bSFull + 2;          // [2]
    static constexpr int bPFull = bSFree + 2;          // [2]
    static constexpr int bPVDone = bPFull + 2;         // [2]
    static constexpr int bFinal = bPVDone + 2;
    static constexpr int kNumBars = bFinal + 1;
    static constexpr uint32_t kMisc = kBar + 8 * kNumBars;        // tmem base, abort flag
    static constexpr uint32_t kBytes = kMisc + 16;
    // 1 KB alignment slack; never below 116 KB so that at most one CTA sits on
    // an SM and its 512 TMEM columns are never contended
    static constexpr uint32_t kAlloc = (kBytes + 1024 > 116u * 1024) ? kBytes + 1024 : 116u * 1024;
    // TMEM columns
    static constexpr uint32_t tS0 = 0, tS1 = 128, tO = 256;
    static constexpr uint32_t tP0 = 256 + HD, tP1 = 256 + HD + 64;
};

struct Ctl {
    uint32_t bar0;           // smem address of barrier 0
    volatile int* abort;
    int* err;
    __device__ uint32_t bar(int i) const { return bar0 + 8u * (uint32_t)i; }
    __device__ bool wait(int i, uint32_t parity) const {
        if (mbar_try(i, parity)) return true;
        const long long t0 = clock64();
        for (;;) {
            if (mbar_try(i, parity)) return true;
            if (*abort) return false;
            if (clock64() - t0 > kWaitLimit) {
                *abort = 1;
                raise_error(err, JANO_ETIMEOUT);
                return false;
            }
        }
    }
    __device__ bool mbar_try(int i, uint32_t parity) const { return ptx::mbar_try_wait(bar(i), parity); }
    // Warp-uniform wait: lane 0 polls, the verdict is broadcast, so the
    // .sync.aligned tcgen05 operations that follow never run divergently.
    __device__ bool warp_wait(int i, uint32_t parity) const {
        int ok = 0;
        if ((threadIdx.x & 31) == 0) ok = wait(i, parity) ? 1 : 0;
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        return ok != 0;
    }
};

template <int HD>
__global__ void __launch_bounds__(kThreads, 1)
attention_kernel(const __grid_constant__ CUtensorMap tmQ,
                 const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV,
                 const int32_t* __restrict__ idx, int n_act, int n_tokens, int heads,
                 float scale_log2, __nv_bfloat16* __restrict__ out, int* err) {
    using L = Layout<HD>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = ptx::smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qt = blockIdx.x, head = blockIdx.y;
    const int q0 = qt * BM;
    const int nt = (n_tokens + BN - 1) / BN;

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
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(ctl.bar(L::bKFull + s), 1);
            ptx::mbar_init(ctl.bar(L::bKEmpty + s), 1);
            ptx::mbar_init(ctl.bar(L::bVFull + s), 1);
            ptx::mbar_init(ctl.bar(L::bVEmpty + s), 1);
        }
        for (int s = 0; s < 2; ++s) {
            ptx::mbar_init(ctl.bar(L::bSFull + s), 1);
            ptx::mbar_init(ctl.bar(L::bSFree + s), 4);
            ptx::mbar_init(ctl.bar(L::bPFull + s), 4);
            ptx::mbar_init(ctl.bar(L::bPVDone + s), 1);
        }
        ptx::mbar_init(ctl.bar(L::bFinal), 1);
        *ctl.abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), 512);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int lastK[kStages], lastV[kStages];
            for (int s = 0; s < kStages; ++s) lastK[s] = lastV[s] = -1;
            ptx::mbar_arrive_expect_tx(ctl.bar(L::bQFull), L::kTile);
            for (int p = 0; p < L::kPanels; ++p)
                ptx::tma_load_3d(base + L::kQ + p * kPanel, &tmQ, ctl.bar(L::bQFull), p * 64, head, q0);
            for (int j = 0; j < nt; ++j) {
                const int st = j % kStages;
                const uint32_t ph = ((j / kStages) & 1) ^ 1;
                if (!ctl.wait(L::bKEmpty + st, ph)) break;
                ptx::mbar_arrive_expect_tx(ctl.bar(L::bKFull + st), L::kTile);
                for (int p = 0; p < L::kPanels; ++p)
                    ptx::tma_load_3d(base + L::kK + st * L::kTile + p * kPanel, &tmK,
                                     ctl.bar(L::bKFull + st), p * 64, head, j * BN);
                lastK[st] = j;
                if (!ctl.wait(L::bVEmpty + st, ph)) break;
                ptx::mbar_arrive_expect_tx(ctl.bar(L::bVFull + st), L::kTile);
                for (int p = 0; p < L::kPanels; ++p)
                    ptx::tma_load_3d(base + L::kV + st * L::kTile + p * kPanel, &tmV,
                                     ctl.bar(L::bVFull + st), p * 64, head, j * BN);
                lastV[st] = j;
            }
            // drain: every copy this CTA issued lands before its smem is released
            ptx::mbar_wait(ctl.bar(L::bQFull), 0, kWaitLimit);
            for (int s = 0; s < kStages; ++s) {
                if (lastK[s] >= 0) ptx::mbar_wait(ctl.bar(L::bKFull + s), (lastK[s] / kStages) & 1, kWaitLimit);
                if (lastV[s] >= 0) ptx::mbar_wait(ctl.bar(L::bVFull + s), (lastV[s] / kStages) & 1, kWaitLimit);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = ptx::idesc_bf16(BM, BN, false, false);
            constexpr uint32_t idesc_pv = ptx::idesc_bf16(BM, HD, false, true);
            bool ok = ctl.wait(L::bQFull, 0);
            auto issue_pv = [&](int i) -> bool {
                const int st = i % kStages, pb = i & 1;
                if (!ctl.wait(L::bPFull + pb, (i >> 1) & 1)) return false;
                if (!ctl.wait(L::bVFull + st, (i / kStages) & 1)) return false;
                ptx::tc_fence_after();
                const uint32_t vbase = base + L::kV + st * L::kTile;
                const uint32_t ptm = tmem + (pb ? L::tP1 : L::tP0);
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    const uint64_t bd = ptx::smem_desc_sw128(vbase + kk * 2048, kPanel, 1024);
                    ptx::mma_ts(tmem + L::tO, ptm + kk * 8, bd, idesc_pv, (i > 0 || kk > 0) ? 1u : 0u);
                }
                ptx::mma_commit(ctl.bar(L::bVEmpty + st));
                ptx::mma_commit(ctl.bar(L::bPVDone + pb));
                return true;
            };
            for (int j = 0; ok && j < nt; ++j) {
                const int st = j % kStages, sb = j & 1;
                if (!ctl.wait(L::bKFull + st, (j / kStages) & 1)) { ok = false; break; }
                if (!ctl.wait(L::bSFree + sb, ((j >> 1) & 1) ^ 1)) { ok = false; break; }
                ptx::tc_fence_after();
                const uint32_t kbase = base + L::kK + st * L::kTile;
                const uint32_t stm = tmem + (sb ? L::tS1 : L::tS0);
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kPanel + (kk & 3) * 32;
                    const uint64_t ad = ptx::smem_desc_sw128(base + L::kQ + off, 16, 1024);
                    const uint64_t bd = ptx::smem_desc_sw128(kbase + off, 16, 1024);
                    ptx::mma_ss(stm, ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
                }
                ptx::mma_commit(ctl.bar(L::bSFull + sb));
                ptx::mma_commit(ctl.bar(L::bKEmpty + st));
                if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
            }
            if (ok) issue_pv(nt - 1);
            // all MMAs of this CTA complete before TMEM can be released
            ptx::mma_commit(ctl.bar(L::bFinal));
            ptx::mbar_wait(ctl.bar(L::bFinal), 0, kWaitLimit);
        }
    } else {
        // ------------------------------------------------------------ softmax
        const int q = warp & 3;                       // TMEM lane quarter of this warp
        const int row = q * 32 + lane;
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        const int qi = q0 + row;
        int t_out = -1;
        if (qi < n_act) {
            t_out = __ldg(idx + qi);
            if (t_out < 0 || t_out >= n_tokens) {
                raise_error(err, JANO_EINDEX);
                t_out = -1;
            }
        }
        float m = -INFINITY, l = 0.f;
        const int tail = n_tokens - (nt - 1) * BN;    // valid keys in the last tile
        bool ok = true;
        for (int j = 0; j < nt; ++j) {
            const int sb = j & 1;
            if (!ctl.warp_wait(L::bSFull + sb, (j >> 1) & 1)) { ok = false; break; }
            ptx::tc_fence_after();
            const uint32_t stm = tmem + lane_off + (sb ? L::tS1 : L::tS0);
            uint32_t s[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) ptx::tmem_ld32(stm + 32 * c, s[c]);
            ptx::tmem_wait_ld();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(ctl.bar(L::bSFree + sb));

            if (j == nt - 1 && tail < BN) {
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (32 * c + e >= tail) s[c][e] = __float_as_uint(-INFINITY);
            }
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int e = 0; e < 32; ++e) mx = fmaxf(mx, __uint_as_float(s[c][e]));
            const float mxs = mx * scale_log2;
            // lazy rescale, decided per warp so the TMEM accesses stay warp-wide:
            // lanes whose max did not grow past 2^8 keep their max (alpha = 1)
            const bool want = mxs > m + 8.0f;
            if (__any_sync(0xFFFFFFFFu, want)) {
                const float m_new = want ? mxs : m;
                if (j > 0) {
                    const float alpha = ptx::ex2(m - m_new);
                    l *= alpha;
                    // O holds PV_0..PV_{j-1}: wait for the last one, rescale in TMEM
                    if (!ctl.warp_wait(L::bPVDone + ((j - 1) & 1), ((j - 1) >> 1) & 1)) { ok = false; break; }
                    ptx::tc_fence_after();
#pragma unroll
                    for (int c = 0; c < HD / 32; ++c) {
                        uint32_t o[32];
                        ptx::tmem_ld32(tmem + lane_off + L::tO + 32 * c, o);
                        ptx::tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        ptx::tmem_st32(tmem + lane_off + L::tO + 32 * c, o);
                    }
                    ptx::tmem_wait_st();
                }
                m = m_new;
            }
            uint32_t p[64];
            float ls = 0.f;
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const float a = ptx::ex2(fmaf(__uint_as_float(s[c][e]), scale_log2, -m));
                    const float b = ptx::ex2(fmaf(__uint_as_float(s[c][e + 1]), scale_log2, -m));
                    ls += a + b;
                    p[c * 16 + e / 2] = ptx::pack_bf16(a, b);
                }
            l += ls;
            // P buffer sb was last read by PV_{j-2}
            if (j >= 2 && !ctl.warp_wait(L::bPVDone + sb, ((j - 2) >> 1) & 1)) { ok = false; break; }
            ptx::tc_fence_after();
            const uint32_t ptm = tmem + lane_off + (sb ? L::tP1 : L::tP0);
            ptx::tmem_st16(ptm, p);
            ptx::tmem_st16(ptm + 16, p + 16);
            ptx::tmem_st16(ptm + 32, p + 32);
            ptx::tmem_st16(ptm + 48, p + 48);
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(ctl.bar(L::bPFull + sb));
        }
        // ------------------------------------------------------------ epilogue
        if (ok && ctl.warp_wait(L::bPVDone + ((nt - 1) & 1), ((nt - 1) >> 1) & 1)) {
            ptx::tc_fence_after();
            const float inv = 1.0f / l;
            __nv_bfloat16* orow = out + ((size_t)(t_out < 0 ? 0 : t_out) * heads + head) * HD;
#pragma unroll
            for (int c = 0; c < HD / 32; ++c) {
                uint32_t o[32];
                ptx::tmem_ld32(tmem + lane_off + L::tO + 32 * c, o);
                ptx::tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    pk[e] = ptx::pack_bf16(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
                if (t_out >= 0) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
                }
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc(tmem, 512);
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

// 3D map over [rows][heads][d] BF16, box = 64 columns x 1 head x 128 rows.
bool make_map(CUtensorMap* m, const void* ptr, int rows, int heads, int d) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)rows};
    const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)heads * d * 2};
    const cuuint32_t box[3] = {64, 1, 128};
    const cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int HD>
cudaError_t launch_hd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                      const int32_t* idx, int n_act, int n_tokens, int heads, float scale,
                      void* out, int* err, cudaStream_t st) {
    using L = Layout<HD>;
    // the shared-memory opt-in is per device: remember which devices have it
    static unsigned long long done_mask = 0;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 64 || !(done_mask & (1ull << dev))) {
        cudaError_t e = cudaFuncSetAttribute(attention_kernel<HD>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kAlloc);
        if (e != cudaSuccess) return e;
        if (dev < 64) done_mask |= 1ull << dev;
    }
    const dim3 grid((n_act + BM - 1) / BM, heads);
    const float scale_log2 = scale * 1.4426950408889634f;
    attention_kernel<HD><<<grid, kThreads, L::kAlloc, st>>>(
        mq, mk, mv, idx, n_act, n_tokens, heads, scale_log2,
        static_cast<__nv_bfloat16*>(out), err);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_active_attention(const void* q, const void* k, const void* v,
                                    const int32_t* idx, int n_act, int n_tokens,
                                    int heads, int d, float scale, void* out,
                                    int* err, cudaStream_t st) {
    if (n_act <= 0) return cudaSuccess;
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, q, n_act, heads, d) || !make_map(&mk, k, n_tokens, heads, d) ||
        !make_map(&mv, v, n_tokens, heads, d))
        return cudaErrorInvalidValue;
    if (d == 128) return launch_hd<128>(mq, mk, mv, idx, n_act, n_tokens, heads, scale, out, err, st);
    return launch_hd<64>(mq, mk, mv, idx, n_act, n_tokens, heads, scale, out, err, st);
}

}  // namespace jano
