// projection.cu -- the DiT block's linear maps on the active tokens only,
// with the rows gathered on the way in and scattered on the way out (Jano
// pages: nl technical summary, Methodologie 2 "KV Cache Mechanisme": per
// step only a subset of the tokens is activated and the K/V of the frozen
// ones are kept, so the Q/K/V and output projections run on the active rows
// alone; zh technical summary 2.2 item 3).
//
//   out_seg(r)[dst_seg(r)][j] = sum_c x[src(r)][c] * w[j][c]
//
// A persistent grid, one CTA per SM, walks the 256-row x BN-column output
// tiles (two 128-row MMA halves that share every weight stage, which cuts
// the shared-memory traffic per FLOP: an SS MMA reads both operands from
// shared memory at 128 B/clk); 9 warps:
//   warps 0-3  producers.  The tile's 256 source rows (src(r) = gather[r],
//            or r) are read once into shared memory.  Per 64-column K block
//            the A rows are gathered with 16-byte cp.async copies (eight
//            lanes per 128-byte row, zero-filled for rows past m), written
//            straight into the 128-byte-swizzled K-major layout the tensor
//            core reads (chunk c of row i at i*128 + ((c ^ (i % 8)) * 16));
//            the weight rows come by one tiled TMA box.  A 3-slot ring; each
//            producer thread hands a stage over with cp.async.mbarrier.arrive
//            (the barrier cannot complete before that thread's copies have
//            landed) plus an ordinary arrive, so it never waits for its own
//            copies and runs as far ahead as the ring allows.
//   warp 4   allocates the 512 TMEM columns; one lane issues tcgen05.mma
//            (kind::f16, M=128, N=BN, K=16, both operands K-major from
//            shared memory, fp32 accumulators in TMEM), two per K slice (one
//            per half of the tile), and frees ring slots with
//            tcgen05.commit.  For BN = 256 one accumulator set (2 x 256
//            columns) fills TMEM; for BN = 128 two sets alternate, so the
//            epilogue overlaps the next tile.
//   warps 5-8  epilogue: thread = one TMEM lane = one row of each half; a
//            tile's accumulators are read 32 columns at a time, rounded to
//            BF16 and stored to the rows' destinations.  The N range may be cut into
//            segments with their own destination and row map, which is how
//            the fused Q/K/V projection writes Q to the active rows and K, V
//            straight into the token-ordered KV cache.
// CTAs are rasterised in groups of 16 row tiles, so one wave of 148 CTAs
// touches about 16 row tiles of x and 9 column tiles of w (both fit in L2).
// Every wait is bounded; on timeout the CTA records JANO_ETIMEOUT, drains its
// copies and MMAs, frees TMEM and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "jano_common.cuh"

namespace jano {
namespace {

constexpr int PM = 256;                 // output rows per tile (two 128-row MMA halves)
constexpr int PK = 64;                  // K columns per stage (128 bytes of BF16)
constexpr int kStages = 3;
constexpr int kProducers = 128;         // warps 0-3
constexpr int kMmaWarp = 4;
constexpr int kThreads = 288;
constexpr int kGroupM = 16;             // row tiles per rasterisation group
constexpr long long kWaitLimit = 1ll << 31;

struct Seg {
    void* dst;                          // BF16 rows of `ld` elements
    const int32_t* rowmap;              // output row of active row r (NULL: r)
    int ld;
    int n_rows;                         // rows of dst (bound for rowmap values)
};

struct GemmArgs {
    const void* x;                      // BF16 [n_x][k]
    const int32_t* gather;              // source row of active row r (NULL: r)
    int m, n_x, n, k;
    int seg_w;                          // columns per segment
    Seg seg[3];
    int* err;
};

template <int BN>
struct PLayout {
    // accumulator sets in TMEM (each: two halves of BN columns): two when
    // they fit in the 512 columns, so the epilogue overlaps the next tile
    static constexpr int kAccBuf = 4 * BN <= 512 ? 2 : 1;
    static constexpr uint32_t kA = PM * PK * 2;                  // 32 KB
    static constexpr uint32_t kB = BN * PK * 2;                  // 32 KB for BN = 256
    static constexpr uint32_t kStage = kA + kB;
    static constexpr uint32_t kBar = kStages * kStage;
    // ring full/empty, accumulator full [2] (MMA commit), accumulator empty
    // [2] (the 4 epilogue warps), the final drain
    static constexpr int bFull = 0, bEmpty = kStages, bAccFull = 2 * kStages,
                         bAccEmpty = bAccFull + 2, bFinal = bAccEmpty + 2, kNumBars = bFinal + 1;
    static constexpr uint32_t kMisc = kBar + 8 * kNumBars;       // tmem base, abort flag
    static constexpr uint32_t kBytes = kMisc + 16;
    static constexpr uint32_t kAlloc = kBytes + 1024;            // slack for 1 KB alignment
    static_assert(kAlloc <= 227 * 1024, "shared memory budget");
};

struct PCtl {
    uint32_t bar0;
    volatile int* abort;
    int* err;
    __device__ uint32_t bar(int i) const { return bar0 + 8u * (uint32_t)i; }
    __device__ bool wait(int i, uint32_t parity) const {
        if (ptx::mbar_try_wait(bar(i), parity)) return true;
        const long long t0 = clock64();
        for (;;) {
            if (ptx::mbar_try_wait(bar(i), parity)) return true;
            if (*abort) return false;
            if (clock64() - t0 > kWaitLimit) {
                *abort = 1;
                raise_error(err, JANO_ETIMEOUT);
                return false;
            }
        }
    }
    __device__ bool warp_wait(int i, uint32_t parity) const {
        int ok = 0;
        if ((threadIdx.x & 31) == 0) ok = wait(i, parity) ? 1 : 0;
        return __shfl_sync(0xFFFFFFFFu, ok, 0) != 0;
    }
};

// 16 bytes global -> shared; `bytes` = 16 copies, 0 writes zeros.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(bytes) : "memory");
}
// Arrive on `bar` once every cp.async this thread issued so far has landed
// (the barrier's pending count is raised first, so the phase waits for it).
__device__ __forceinline__ void cp_async_arrive(uint32_t bar) {
    asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// Order shared-memory writes this thread has observed (through an mbarrier)
// before its following async-proxy accesses (the tensor core's operand reads).
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, uint32_t bar, int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar), "r"(c0), "r"(c1) : "memory");
}

// Output tile number t of the grouped rasterisation: consecutive tiles walk
// the column tiles of a group of kGroupM row tiles.
__device__ __forceinline__ void tile_coords(int t, int m_tiles, int n_tiles, int& m_tile, int& n_tile) {
    const int per_group = kGroupM * n_tiles;
    const int group = t / per_group;
    const int first_m = group * kGroupM;
    const int gm = min(kGroupM, m_tiles - first_m);
    m_tile = first_m + (t % per_group) % gm;
    n_tile = (t % per_group) / gm;
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
projection_kernel(const __grid_constant__ CUtensorMap tmB, const __grid_constant__ GemmArgs a) {
    using L = PLayout<BN>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = ptx::smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const int n_tiles = (a.n + BN - 1) / BN;
    const int m_tiles = (a.m + PM - 1) / PM;
    const int tiles = n_tiles * m_tiles;
    const int nkb = (a.k + PK - 1) / PK;

    PCtl ctl;
    ctl.bar0 = base + L::kBar;
    ctl.abort = reinterpret_cast<volatile int*>(gbase + L::kMisc + 4);
    ctl.err = a.err;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + L::kMisc);

    if (threadIdx.x == 0) {
        ptx::prefetch_tmap(&tmB);
        for (int s = 0; s < kStages; ++s) {
            // every producer thread once (A) plus the weight copy's expect_tx
            ptx::mbar_init(ctl.bar(L::bFull + s), kProducers + 1);
            ptx::mbar_init(ctl.bar(L::bEmpty + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(ctl.bar(L::bAccFull + b), 1);
            ptx::mbar_init(ctl.bar(L::bAccEmpty + b), 4);
        }
        ptx::mbar_init(ctl.bar(L::bFinal), 1);
        *ctl.abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), 512);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp < kProducers / 32) {
        // ------------------------------------------------------------ producers
        const int t = threadIdx.x;
        const int c = t & 7;                          // 16-byte chunk of a 128-byte row
        const int rg = t >> 3;                        // first row (rows rg, rg+16, ...)
        const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(a.x);
        int q = 0;                                    // stage counter, across tiles
        bool ok = true;
        for (int tile = blockIdx.x; ok && tile < tiles; tile += gridDim.x) {
            int mt, nt;
            tile_coords(tile, m_tiles, n_tiles, mt, nt);
            const int m0 = mt * PM, n0 = nt * BN;
            // this thread's 8 source rows; rows past m and bad indices copy zeros
            int src[PM / 16];
#pragma unroll
            for (int u = 0; u < PM / 16; ++u) {
                const int r = m0 + rg + 16 * u;
                int sr = -1;
                if (r < a.m) {
                    sr = a.gather ? __ldg(a.gather + r) : r;
                    if (sr < 0 || sr >= a.n_x) {
                        if (nt == 0) raise_error(a.err, JANO_EINDEX);
                        sr = -1;
                    }
                }
                src[u] = sr;
            }
            for (int kb = 0; kb < nkb; ++kb, ++q) {
                const int s = q % kStages;
                // warp-uniform: lane 0 waits, the warp follows
                if (!ctl.warp_wait(L::bEmpty + s, ((q / kStages) & 1) ^ 1)) { ok = false; break; }
                const uint32_t sa = base + s * L::kStage;
                const uint32_t full = ctl.bar(L::bFull + s);
#ifdef JANO_INJECT_DROP_LOAD
                // failure-path test builds only: stage q's weight copy is never
                // issued, so the MMA's bounded wait for it runs out (JANO_ETIMEOUT)
                if (t == 0 && q != JANO_INJECT_DROP_LOAD) {
#else
                if (t == 0) {
#endif
                    ptx::mbar_arrive_expect_tx(full, L::kB);
                    tma_load_2d(sa + L::kA, &tmB, full, kb * PK, n0);
                }
                const int col = kb * PK + 8 * c;      // first element of this thread's chunk
                const bool in_k = col < a.k;
#pragma unroll
                for (int u = 0; u < PM / 16; ++u) {
                    const int i = rg + 16 * u;        // row of the tile
                    const bool live = src[u] >= 0 && in_k;
                    const void* g = live ? static_cast<const void*>(xb + (size_t)src[u] * a.k + col) : a.x;
                    cp_async16(sa + i * 128 + ((c ^ (i & 7)) << 4), g, live ? 16u : 0u);
                }
                cp_async_arrive(full);
                ptx::mbar_arrive(full);
            }
        }
        // no copy outlives the CTA (after a timeout some stages are never consumed)
        cp_async_wait_all();
        if (t == 0) {
            // drain: every weight copy this CTA issued lands before its smem is released
            for (int r = (q > kStages ? q - kStages : 0); r < q; ++r)
                ptx::mbar_wait(ctl.bar(L::bFull + r % kStages), (r / kStages) & 1, kWaitLimit);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = ptx::idesc_bf16(128, BN, false, false);
            int q = 0, lt = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < tiles; tile += gridDim.x, ++lt) {
                const int b = lt % L::kAccBuf;
                // the epilogue has read this accumulator set's previous tile
                if (!ctl.wait(L::bAccEmpty + b, ((lt / L::kAccBuf) & 1) ^ 1)) { ok = false; break; }
                ptx::tc_fence_after();
                const uint32_t acc = tmem + b * 2 * BN;       // rows 0-127; rows 128-255 at + BN
                for (int kb = 0; kb < nkb; ++kb, ++q) {
                    const int s = q % kStages;
                    if (!ctl.wait(L::bFull + s, (q / kStages) & 1)) { ok = false; break; }
                    fence_proxy_async();
                    ptx::tc_fence_after();
                    const uint32_t sa = base + s * L::kStage;
                    // both 128-row halves of A against the same B stage
#pragma unroll
                    for (int kk = 0; kk < PK / 16; ++kk) {
                        const uint64_t bd = ptx::smem_desc_sw128(sa + L::kA + kk * 32, 16, 1024);
                        const uint32_t accum = (kb > 0 || kk > 0) ? 1u : 0u;
                        ptx::mma_ss(acc, ptx::smem_desc_sw128(sa + kk * 32, 16, 1024), bd, idesc, accum);
                        ptx::mma_ss(acc + BN, ptx::smem_desc_sw128(sa + 128 * 128 + kk * 32, 16, 1024), bd,
                                    idesc, accum);
                    }
                    ptx::mma_commit(ctl.bar(L::bEmpty + s));
                }
                if (ok) ptx::mma_commit(ctl.bar(L::bAccFull + b));
            }
            // every MMA of this CTA completes before TMEM is released
            ptx::mma_commit(ctl.bar(L::bFinal));
            ptx::mbar_wait(ctl.bar(L::bFinal), 0, kWaitLimit);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int qd = warp & 3;                      // TMEM lane quarter of this warp
        int lt = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++lt) {
            const int b = lt % L::kAccBuf;
            if (!ctl.warp_wait(L::bAccFull + b, (lt / L::kAccBuf) & 1) || *ctl.abort) break;
            ptx::tc_fence_after();
            int mt, nt;
            tile_coords(tile, m_tiles, n_tiles, mt, nt);
            const int m0 = mt * PM, n0 = nt * BN;
            const int seg_i = n0 / a.seg_w;
            const Seg& sg = a.seg[seg_i];
            const int col0 = n0 - seg_i * a.seg_w;    // first column of the tile in its segment
            const int cols = min(BN, a.seg_w - col0);  // columns of this tile inside the segment
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                const int r = m0 + 128 * half + qd * 32 + lane;
                int dst_row = -1;
                if (r < a.m) {
                    dst_row = sg.rowmap ? __ldg(sg.rowmap + r) : r;
                    // scattered rows: in range and strictly ascending
                    if (dst_row < 0 || dst_row >= sg.n_rows ||
                        (sg.rowmap && r > 0 && __ldg(sg.rowmap + r - 1) >= dst_row)) {
                        raise_error(a.err, JANO_EINDEX);
                        dst_row = -1;
                    }
                }
                const uint32_t taddr = tmem + (b * 2 + half) * BN + ((uint32_t)(qd * 32) << 16);
                __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(sg.dst) +
                                      (size_t)(dst_row < 0 ? 0 : dst_row) * sg.ld + col0;
#pragma unroll 1
                for (int cc = 0; cc < BN / 32; ++cc) {
                    uint32_t v[32];
                    ptx::tmem_ld32(taddr + 32 * cc, v);
                    ptx::tmem_wait_ld();
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        pk[e] = ptx::pack_bf16(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
                    if (dst_row >= 0) {
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            if (32 * cc + 8 * u < cols)
                                *reinterpret_cast<uint4*>(orow + 32 * cc + 8 * u) =
                                    make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
                    }
                }
            }
            // this accumulator set may take the next tile
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(ctl.bar(L::bAccEmpty + b));
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == kMmaWarp) ptx::tmem_dealloc(tmem, 512);
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

// 2-D BF16 map over [rows][cols] (cols contiguous), box = 64 columns x box_rows.
bool make_map2d(CUtensorMap* m, const void* ptr, int rows, int cols, int box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {(cuuint32_t)PK, (cuuint32_t)box_rows};
    const cuuint32_t es[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN>
cudaError_t launch_bn(const void* w, const GemmArgs& a, cudaStream_t st) {
    using L = PLayout<BN>;
    CUtensorMap mB;
    if (!make_map2d(&mB, w, a.n, a.k, BN)) return cudaErrorInvalidValue;
    static DeviceOnce opted_in;   // per-device shared-memory opt-in
    int dev = 0;
    cudaGetDevice(&dev);
    if (!opted_in.done(dev)) {
        cudaError_t e = cudaFuncSetAttribute(projection_kernel<BN>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kAlloc);
        if (e != cudaSuccess) return e;
        opted_in.mark(dev);
    }
    const int tiles = ((a.m + PM - 1) / PM) * ((a.n + BN - 1) / BN);
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = tiles < sms ? tiles : sms;      // persistent: one CTA per SM
    projection_kernel<BN><<<grid, kThreads, L::kAlloc, st>>>(mB, a);
    return cudaGetLastError();
}

}  // namespace

// Column tile width for a segment width: 256 when it divides the segments
// (or there is one segment), else 128; 0 if neither fits.
int projection_tile_n(int n, int seg_w, int n_seg) {
    if (n_seg == 1) return n >= 256 ? 256 : 128;
    if (seg_w % 256 == 0) return 256;
    if (seg_w % 128 == 0) return 128;
    return 0;
}

cudaError_t launch_projection(const void* x, int n_x, const int32_t* gather, int m, const void* w,
                              int n, int k, int n_seg, const ProjSeg* segs, int* err,
                              cudaStream_t st) {
    if (m <= 0) return cudaSuccess;
    GemmArgs a{};
    a.x = x;
    a.gather = gather;
    a.m = m;
    a.n_x = n_x;
    a.n = n;
    a.k = k;
    a.seg_w = n / n_seg;
    for (int i = 0; i < n_seg; ++i) {
        a.seg[i].dst = segs[i].dst;
        a.seg[i].rowmap = segs[i].rowmap;
        a.seg[i].ld = segs[i].ld;
        a.seg[i].n_rows = segs[i].n_rows;
    }
    a.err = err;
    const int bn = projection_tile_n(n, a.seg_w, n_seg);
    if (bn == 256) return launch_bn<256>(w, a, st);
    if (bn == 128) return launch_bn<128>(w, a, st);
    return cudaErrorInvalidValue;
}

}  // namespace jano
