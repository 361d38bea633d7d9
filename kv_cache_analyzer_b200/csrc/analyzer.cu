// analyzer.cu -- block-wise complexity analyzer (Jano pages: zh technical
// summary 2.1; nl technical summary, Methodologie 1 "Implementatie"; pt 2.A).
//
//   S_b = mean over k=1..K-1, c, (f,h,w) in b of
//         |x_{k+1} - 2x_k + x_{k-1}| + w_t |D_f x_k| + w_s sqrt(D_h x_k^2 + D_w x_k^2)
//
// HBM-bound streaming stencil.  The latent history [K+1][C][F][H][W] is cut
// into work units of one frame-block x one block-row x a chunk of Wc columns
// (a whole number of blocks).  A persistent grid walks the units; in each
// CTA one producer thread streams, for every channel of the unit, a stage of
// two TMA boxes into a shared-memory ring:
//   A  all K+1 snapshots of the unit's rows plus the h+1 halo row and 4
//      extra columns (the w+1 neighbours), box (Wc+4, bh+1, bf, 1, K+1);
//   B  snapshots 1..K-1 of the next frame's rows (the f+1 neighbours of the
//      block's last frame), box (Wc, bh, 1, 1, K-1).
// Out-of-range rows, columns and frames arrive zero-filled and are masked
// in the arithmetic.  All compute threads work on the same stage: thread
// (k, row, 4 columns) evaluates the stencil at step k from shared memory with
// 128-bit loads and keeps its sums over the channels in registers, so the
// ring can run several stages ahead of the arithmetic.  At the end of a unit
// the per-thread sums are added per block over k, rows and columns in a
// fixed order (deterministic, no atomics).
// Every byte of the latent is read from HBM once; neighbour rows and frames
// come back from L2.
//
// The literal reading (second differences over the steps of the gradients,
//   w_t |D2 D_f x| + w_s sqrt((D2 D_h x)^2 + (D2 D_w x)^2),  D2 y = y_{k+1} - 2y_k + y_{k-1})
// runs the same pipeline with box B widened to snapshots 0..K: since D2 and
// the forward differences commute, a thread forms D2 x at its element and at
// the f+1, h+1, w+1 neighbours and takes their differences.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "jano_common.cuh"

namespace jano {
namespace {

constexpr int kMaxStages = 16;
// float4 vectors (4 consecutive columns each) per thread and step
#ifndef JANO_ANALYZER_VEC
#define JANO_ANALYZER_VEC 1
#endif
constexpr int kVec = JANO_ANALYZER_VEC;
constexpr long long kWaitLimit = 1ll << 31;
// Unit width in columns (measured best on the large video latent: 80, i.e.
// two units per 160-column row) and the shared-memory budget per CTA in KB
// (0: the smallest of 72 / 110 / 220 KB that holds a ring of >= 4 stages;
// 72 KB gives three CTAs per SM).
#ifndef JANO_ANALYZER_WC
#define JANO_ANALYZER_WC 80
#endif
#ifndef JANO_ANALYZER_SMEM_KB
#define JANO_ANALYZER_SMEM_KB 0
#endif

struct AGeo {
    int K, C, F, H, W;
    int bf, bh, bw;
    int nBh, nBw;
    int Wc;                // columns per unit, multiple of 4 and of bw
    int n_wc;              // units along W
    int n_units;
    int NP;                // positions per step: rows x Wc/4
    int NC;                // compute threads: NP x (K-1), rounded up to 32
    int S;                 // ring stages
    int stage_bytes;       // per channel stage, 128-byte multiple
    int bytesA, bytesB;    // TMA transaction bytes of boxes A and B
    int offB;              // byte offset of box B in a stage (128-aligned)
    int red_off;           // offset of the reduction area [K-1][R][Wc]
    int smem;              // dynamic shared memory bytes
    int LA;                // floats per staged row of box A (Wc + 4)
    float w_t, w_s;
};

__device__ __forceinline__ float term(float d2, float df, float dh, float dw, float w_t, float w_s) {
    return fabsf(d2) + w_t * fabsf(df) + w_s * ptx::sqrt_approx(fmaf(dh, dh, dw * dw));
}

// Bounded wait that also gives up as soon as another thread of the CTA has
// recorded a timeout (abort flag in shared memory).  It polls rather than
// suspends: every stage's hand-off is on the ring's critical path, and the
// compute warps have nothing else to issue meanwhile (measured 3% faster).
__device__ __forceinline__ bool bounded_wait(uint32_t bar, uint32_t parity, int* err,
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

__device__ __forceinline__ void tma_load_5d(uint32_t dst, const void* tmap, uint32_t bar,
                                            int c0, int c1, int c2, int c3, int c4) {
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar),
          "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4) : "memory");
}

__device__ __forceinline__ void named_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ float4 d2_of(const float* A, int o, int kA) {
    const float4 m = *reinterpret_cast<const float4*>(A + o - kA);
    const float4 z = *reinterpret_cast<const float4*>(A + o);
    const float4 p = *reinterpret_cast<const float4*>(A + o + kA);
    return make_float4(p.x - 2.f * z.x + m.x, p.y - 2.f * z.y + m.y, p.z - 2.f * z.z + m.z,
                       p.w - 2.f * z.w + m.w);
}

__device__ __forceinline__ float lit_term(float gf, float gh, float gw, float w_t, float w_s) {
    return w_t * fabsf(gf) + w_s * ptx::sqrt_approx(fmaf(gh, gh, gw * gw));
}

// kLit: the literal reading (see the file comment).
template <bool kLit>
__global__ void __launch_bounds__(1024)
analyzer_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                AGeo g, float* __restrict__ scores, int* err) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = ptx::smem_u32(smem_raw);
    const uint32_t base = (raw + 127u) & ~127u;
    uint8_t* gbase = smem_raw + (base - raw);
    const int S = g.S;
    const uint32_t bar_full = base + (uint32_t)g.red_off - 16u * S - 16u;   // S full, S empty barriers
    volatile int* abort = reinterpret_cast<volatile int*>(gbase + g.red_off - 16);
    auto full = [&](int s) { return bar_full + 8u * s; };
    auto empty = [&](int s) { return bar_full + 8u * (S + s); };
    float* red = reinterpret_cast<float*>(gbase + g.red_off);         // [K-1][R][Wc]
    const int R = g.bf * g.bh;
    const int n_compute = g.NC;

    if (threadIdx.x == 0) {
        ptx::prefetch_tmap(&tmA);
        ptx::prefetch_tmap(&tmB);
        for (int s = 0; s < S; ++s) {
            ptx::mbar_init(full(s), 1);
            ptx::mbar_init(empty(s), n_compute / 32);
        }
        *abort = 0;
        ptx::fence_mbar_init();
    }
    __syncthreads();

    const int tid = threadIdx.x;
    if (tid >= n_compute) {
        // ------------------------------------------------------------ producer
        if (tid == n_compute) {
            int last[kMaxStages];                 // phase of the last copy into each slot
            for (int q = 0; q < S; ++q) last[q] = -1;
            int slot = 0, phase = 0;              // ring position, advanced incrementally
            bool ok = true;
            for (int u = blockIdx.x; ok && u < g.n_units; u += gridDim.x) {
                const int wc = u % g.n_wc;
                const int hb = (u / g.n_wc) % g.nBh;
                const int fb = u / (g.n_wc * g.nBh);
                const int f0 = fb * g.bf, h0 = hb * g.bh, w0 = wc * g.Wc;
                const bool has_next = f0 + g.bf < g.F;
                for (int c = 0; c < g.C; ++c) {
                    if (!bounded_wait(empty(slot), (uint32_t)(phase ^ 1), err, abort)) { ok = false; break; }
                    const uint32_t dst = base + (uint32_t)slot * g.stage_bytes;
                    ptx::mbar_arrive_expect_tx(full(slot), g.bytesA + (has_next ? g.bytesB : 0));
                    tma_load_5d(dst, &tmA, full(slot), w0, h0, f0, c, 0);
                    if (has_next)
                        tma_load_5d(dst + g.offB, &tmB, full(slot), w0, h0, f0 + g.bf, c, kLit ? 0 : 1);
                    last[slot] = phase;
                    if (++slot == S) { slot = 0; phase ^= 1; }
                }
            }
            // drain: the copies this CTA issued land before its smem is released
            for (int q = 0; q < S; ++q)
                if (last[q] >= 0) ptx::mbar_wait(full(q), (uint32_t)last[q], kWaitLimit);
        }
        return;
    }

    // ---------------------------------------------------------------- compute
    const int lane = tid & 31;
    const int Wv = g.Wc / (4 * kVec);              // thread columns (kVec float4 each)
    const int k = 1 + tid / g.NP;                  // step of this thread (1..K-1; >= K: idle)
    const int pos = tid % g.NP;
    const int r = pos / Wv, wv = pos % Wv;
    const int fr = r / g.bh, hr = r % g.bh;
    const int LA = g.LA;                           // floats per staged row of box A
    const int rowsA = g.bh + 1;
    const int wr = 4 * kVec * wv;
    // float offsets inside a stage, fixed for the whole kernel
    const int o_x0 = ((k * g.bf + fr) * rowsA + hr) * LA + wr;
    const int o_xm = o_x0 - g.bf * rowsA * LA;
    const int o_xp = o_x0 + g.bf * rowsA * LA;
    const int o_nh = o_x0 + LA;
    const int o_nf = fr + 1 < g.bf ? o_x0 + rowsA * LA : g.offB / 4 + ((k - 1) * g.bh + hr) * g.Wc + wr;
    // literal reading: snapshot stride inside box A, and the f+1 neighbour at
    // snapshot k with its own snapshot stride (box B then holds 0..K)
    const int kA = g.bf * rowsA * LA;
    const bool nf_in_A = fr + 1 < g.bf;
    const int o_nf_lit = nf_in_A ? o_x0 + rowsA * LA : g.offB / 4 + (k * g.bh + hr) * g.Wc + wr;
    const int kF_lit = nf_in_A ? kA : g.bh * g.Wc;
    int slot = 0, phase = 0;                       // ring position, advanced incrementally
    for (int u = blockIdx.x; u < g.n_units; u += gridDim.x) {
        const int wc = u % g.n_wc;
        const int hb = (u / g.n_wc) % g.nBh;
        const int fb = u / (g.n_wc * g.nBh);
        const int f0 = fb * g.bf, h0 = hb * g.bh, w0 = wc * g.Wc;
        const int f = f0 + fr, h = h0 + hr, w = w0 + wr;
        const bool act = k < g.K && f < g.F && h < g.H && w < g.W;
        const bool has_f = f + 1 < g.F, has_h = h + 1 < g.H;
        float acc[4 * kVec];
#pragma unroll
        for (int e = 0; e < 4 * kVec; ++e) acc[e] = 0.f;
        for (int c = 0; c < g.C; ++c) {
            // after a timeout the CTA stops computing but keeps meeting its barriers
            const bool ready = bounded_wait(full(slot), (uint32_t)phase, err, abort);
            if (ready && act) {
                const float* A = reinterpret_cast<const float*>(gbase + (size_t)slot * g.stage_bytes);
                if constexpr (kLit) {
#pragma unroll
                    for (int v = 0; v < kVec; ++v) {
                        const float4 d = d2_of(A, o_x0 + 4 * v, kA);
                        const float4 dh = has_h ? d2_of(A, o_nh + 4 * v, kA) : d;
                        const float4 df = has_f ? d2_of(A, o_nf_lit + 4 * v, kF_lit) : d;
                        // w+1 neighbour of the 4th element (dropped past the tensor)
                        const int ow = o_x0 + 4 * v + 4;
                        const float dw = (w + 4 * v + 4 < g.W) ? A[ow + kA] - 2.f * A[ow] + A[ow - kA] : d.w;
                        float* a = acc + 4 * v;
                        a[0] += lit_term(df.x - d.x, dh.x - d.x, d.y - d.x, g.w_t, g.w_s);
                        a[1] += lit_term(df.y - d.y, dh.y - d.y, d.z - d.y, g.w_t, g.w_s);
                        a[2] += lit_term(df.z - d.z, dh.z - d.z, d.w - d.z, g.w_t, g.w_s);
                        a[3] += lit_term(df.w - d.w, dh.w - d.w, dw - d.w, g.w_t, g.w_s);
                    }
                } else {
#pragma unroll
                    for (int v = 0; v < kVec; ++v) {
                        const float4 x0 = *reinterpret_cast<const float4*>(A + o_x0 + 4 * v);
                        const float4 xm = *reinterpret_cast<const float4*>(A + o_xm + 4 * v);
                        const float4 xp = *reinterpret_cast<const float4*>(A + o_xp + 4 * v);
                        const float4 nh = has_h ? *reinterpret_cast<const float4*>(A + o_nh + 4 * v) : x0;
                        const float4 nf = has_f ? *reinterpret_cast<const float4*>(A + o_nf + 4 * v) : x0;
                        // w+1 neighbour of the 4th element; zero-filled beyond the tensor, and the
                        // difference is dropped there (w + 4v + 4 >= W)
                        const float nx = A[o_x0 + 4 * v + 4];
                        const float nw = (w + 4 * v + 4 < g.W) ? nx : x0.w;
                        float* a = acc + 4 * v;
                        a[0] += term(xp.x - 2.f * x0.x + xm.x, nf.x - x0.x, nh.x - x0.x, x0.y - x0.x, g.w_t, g.w_s);
                        a[1] += term(xp.y - 2.f * x0.y + xm.y, nf.y - x0.y, nh.y - x0.y, x0.z - x0.y, g.w_t, g.w_s);
                        a[2] += term(xp.z - 2.f * x0.z + xm.z, nf.z - x0.z, nh.z - x0.z, x0.w - x0.z, g.w_t, g.w_s);
                        a[3] += term(xp.w - 2.f * x0.w + xm.w, nf.w - x0.w, nh.w - x0.w, nw - x0.w, g.w_t, g.w_s);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(empty(slot));
            if (++slot == S) { slot = 0; phase ^= 1; }
        }
        // this thread's sums -> red[k-1][r][wr ..] (zeros where inactive or past W)
        if (k < g.K) {
            float* dst = red + ((size_t)(k - 1) * R + r) * g.Wc + wr;
#pragma unroll
            for (int e = 0; e < 4 * kVec; ++e) dst[e] = (act && w + e < g.W) ? acc[e] : 0.f;
        }
        named_sync(1, n_compute);
        const int nb = g.Wc / g.bw;
        for (int ob = tid; ob < nb; ob += n_compute) {
            const int ws = w0 + ob * g.bw;
            if (ws >= g.W) continue;
            const int cols = min(g.bw, g.W - ws);
            const int rows_f = min(g.bf, g.F - f0), rows_h = min(g.bh, g.H - h0);
            float sum = 0.f;
            for (int kk = 0; kk < g.K - 1; ++kk)
                for (int rr = 0; rr < R; ++rr) {
                    const float* src = red + ((size_t)kk * R + rr) * g.Wc + ob * g.bw;
                    for (int e = 0; e < g.bw; ++e) sum += src[e];
                }
            const float cnt = (float)(g.K - 1) * (float)g.C * (float)(rows_f * rows_h * cols);
            scores[((size_t)fb * g.nBh + hb) * g.nBw + (ws / g.bw)] = sum / cnt;
        }
        named_sync(1, n_compute);
    }
}

// ---------------------------------------------------------------------------
// Frame-group form: the default reading with K = 5 and blocks of one frame,
// at most 4 rows (1, 2 or 4) and 1-32 columns (a power of two) -- every
// workload of the pages' configurations.  A work unit is G consecutive
// frames x 4 rows x Wc columns (Wc a multiple of 32); its stage per channel
// is box A (all K+1 snapshots of the G frames, the 4 rows and the h+1 halo
// row, Wc + 4 columns) and box B (the frame after the group, 4 rows,
// snapshots 1..K-1).  Only the group's last frame takes its f+1 neighbour
// from box B; the others find it in box A, so the bytes each stage brings
// from L2 per frame fall with G (on the large video latent: 177 MB for the
// 116 MB read once from HBM, against 235 MB with one frame per unit).
// Warp = one frame x 4 rows x 32 columns, lane = (row, float4), so a
// quarter-warp reads 128 consecutive bytes of one staged row.  Each thread
// evaluates all K-1 steps of its 4 columns per stage (its K+1 snapshots in
// registers, the neighbours read as each step needs them) and the warp
// frees the slot after the arithmetic; at 64 registers a thread, several
// small CTAs share an SM, each with a short ring of its own.  At the end of a unit
// the block sums are formed by warp shuffles (xor butterflies over the rows
// of a block and, for blocks wider than 4 columns, over its float4 lanes):
// each partner pair adds the same two values, so every lane of a block ends
// with the same bits whatever the scheduling (deterministic).
struct FGeo {
    int C, F, H, W;
    int bh, bw, nBh, nBw;
    int G, Wc, LA;                 // frames and columns per unit, staged row length (Wc + 4)
    int n_wc, n_rg, n_units;       // units along W, row groups of 4 along H, all units
    int n_warps;                   // compute warps: G x Wc / 32
    int S, stage_bytes, bytesA, bytesB, offB, smem;
    float w_t, w_s;
};

#ifndef JANO_ANALYZER_FG
#define JANO_ANALYZER_FG 1
#endif
constexpr int kFgMaxThreads = 512;

template <int K>
__global__ void __launch_bounds__(kFgMaxThreads)
analyzer_fg_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   FGeo g, float* __restrict__ scores, int* err) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = ptx::smem_u32(smem_raw);
    const uint32_t base = (raw + 127u) & ~127u;
    uint8_t* gbase = smem_raw + (base - raw);
    const int S = g.S;
    const uint32_t bars = base + (uint32_t)(S * g.stage_bytes);        // S full, S empty barriers
    volatile int* abort = reinterpret_cast<volatile int*>(gbase + S * g.stage_bytes + 16 * S);
    auto full = [&](int s) { return bars + 8u * s; };
    auto empty = [&](int s) { return bars + 8u * (S + s); };
    const int n_compute = g.n_warps * 32;

    if (threadIdx.x == 0) {
        ptx::prefetch_tmap(&tmA);
        ptx::prefetch_tmap(&tmB);
        for (int s = 0; s < S; ++s) {
            ptx::mbar_init(full(s), 1);
            ptx::mbar_init(empty(s), g.n_warps);
        }
        *abort = 0;
        ptx::fence_mbar_init();
    }
    __syncthreads();

    const int tid = threadIdx.x;
    if (tid >= n_compute) {
        // ------------------------------------------------------------ producer
        if (tid == n_compute) {
            int last[kMaxStages];                 // phase of the last copy into each slot
            for (int q = 0; q < S; ++q) last[q] = -1;
            int slot = 0, phase = 0;
            bool ok = true;
            for (int u = blockIdx.x; ok && u < g.n_units; u += gridDim.x) {
                const int wc = u % g.n_wc;
                const int rg = (u / g.n_wc) % g.n_rg;
                const int fg = u / (g.n_wc * g.n_rg);
                const int f0 = fg * g.G, h0 = rg * 4, w0 = wc * g.Wc;
                const bool has_next = f0 + g.G < g.F;
                for (int c = 0; c < g.C; ++c) {
                    if (!bounded_wait(empty(slot), (uint32_t)(phase ^ 1), err, abort)) { ok = false; break; }
                    const uint32_t dst = base + (uint32_t)slot * g.stage_bytes;
                    ptx::mbar_arrive_expect_tx(full(slot), g.bytesA + (has_next ? g.bytesB : 0));
                    tma_load_5d(dst, &tmA, full(slot), w0, h0, f0, c, 0);
                    if (has_next) tma_load_5d(dst + g.offB, &tmB, full(slot), w0, h0, f0 + g.G, c, 1);
                    last[slot] = phase;
                    if (++slot == S) { slot = 0; phase ^= 1; }
                }
            }
            for (int q = 0; q < S; ++q)
                if (last[q] >= 0) ptx::mbar_wait(full(q), (uint32_t)last[q], kWaitLimit);
        }
        return;
    }

    // ---------------------------------------------------------------- compute
    const int warp = tid >> 5, lane = tid & 31;
    const int wpf = g.Wc >> 5;                         // warps per frame
    const int fr = warp / wpf;                         // frame inside the group
    const int hr = lane >> 3;                          // row inside the unit
    const int wr = ((warp % wpf) << 5) + ((lane & 7) << 2);   // first column inside the unit
    const int LA = g.LA;
    // float offsets inside a stage: this row at snapshot 0, the snapshot
    // stride of box A, and the f+1 neighbour (box A, or box B for the
    // group's last frame) as base + k * stride for snapshot k
    const int oA = (fr * 5 + hr) * LA + wr;
    const int sA = g.G * 5 * LA;
    const bool nf_in_A = fr + 1 < g.G;
    const int oF = nf_in_A ? oA + 5 * LA : g.offB / 4 + hr * g.Wc + wr - 4 * g.Wc;
    const int sF = nf_in_A ? sA : 4 * g.Wc;
    const float w_t = g.w_t, w_s = g.w_s;
    int slot = 0, phase = 0;
    for (int u = blockIdx.x; u < g.n_units; u += gridDim.x) {
        const int wc = u % g.n_wc;
        const int rg = (u / g.n_wc) % g.n_rg;
        const int fg = u / (g.n_wc * g.n_rg);
        const int f = fg * g.G + fr, h = rg * 4 + hr, w = wc * g.Wc + wr;
        const bool act = f < g.F && h < g.H && w < g.W;      // W is a multiple of 4
        const bool has_f = f + 1 < g.F, has_h = h + 1 < g.H, has_w = w + 4 < g.W;
        // a warp whose lanes all have every neighbour takes the unmasked path
        const bool interior = __all_sync(0xFFFFFFFFu, act && has_f && has_h && has_w);
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
        for (int c = 0; c < g.C; ++c) {
            const bool ready = bounded_wait(full(slot), (uint32_t)phase, err, abort);
            if (ready && act) {
                const float* A = reinterpret_cast<const float*>(gbase + (size_t)slot * g.stage_bytes);
                float4 x[K + 1];
#pragma unroll
                for (int s = 0; s <= K; ++s) x[s] = *reinterpret_cast<const float4*>(A + oA + s * sA);
#pragma unroll
                for (int k = 1; k < K; ++k) {
                    const float4 xm = x[k - 1], x0 = x[k], xp = x[k + 1];
                    float4 nhk = *reinterpret_cast<const float4*>(A + oA + k * sA + LA);
                    float4 nfk = *reinterpret_cast<const float4*>(A + oF + k * sF);
                    float nxk = A[oA + k * sA + 4];
                    if (!interior) {
                        if (!has_h) nhk = x0;
                        if (!has_f) nfk = x0;
                        if (!has_w) nxk = x0.w;
                    }
                    a0 += term(xp.x - 2.f * x0.x + xm.x, nfk.x - x0.x, nhk.x - x0.x, x0.y - x0.x, w_t, w_s);
                    a1 += term(xp.y - 2.f * x0.y + xm.y, nfk.y - x0.y, nhk.y - x0.y, x0.z - x0.y, w_t, w_s);
                    a2 += term(xp.z - 2.f * x0.z + xm.z, nfk.z - x0.z, nhk.z - x0.z, x0.w - x0.z, w_t, w_s);
                    a3 += term(xp.w - 2.f * x0.w + xm.w, nfk.w - x0.w, nhk.w - x0.w, nxk - x0.w, w_t, w_s);
                }
            }
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(empty(slot));
            if (++slot == S) { slot = 0; phase ^= 1; }
        }
        // ---- block sums by warp shuffles (bh, bw uniform: no divergence)
        float p[4] = {a0, a1, a2, a3};
        int nbt = 4;                                   // block partials per thread
        if (g.bw >= 4) { p[0] = (a0 + a1) + (a2 + a3); nbt = 1; }
        else if (g.bw == 2) { p[0] = a0 + a1; p[1] = a2 + a3; nbt = 2; }
        for (int o = 8; o < 8 * g.bh; o <<= 1) {       // over the block's rows
#pragma unroll
            for (int j = 0; j < 4; ++j) p[j] += __shfl_xor_sync(0xFFFFFFFFu, p[j], o);
        }
        for (int o = 1; o < g.bw / 4; o <<= 1) p[0] += __shfl_xor_sync(0xFFFFFFFFu, p[0], o);
        const bool writer = act && hr % g.bh == 0 && (g.bw <= 4 || ((lane & 7) & (g.bw / 4 - 1)) == 0);
        if (writer) {
            const int hb = h / g.bh;
            const int rows = min(g.bh, g.H - hb * g.bh);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int ws = w + j * g.bw;
                if (j >= nbt || ws >= g.W) break;
                const int wb = ws / g.bw;
                const int cols = min(g.bw, g.W - wb * g.bw);
                const float cnt = (float)(K - 1) * (float)g.C * (float)(rows * cols);
                scores[((size_t)f * g.nBh + hb) * g.nBw + wb] = p[j] / cnt;
            }
        }
    }
}

int gcd(int a, int b) {
    while (b) { const int t = a % b; a = b; b = t; }
    return a;
}

int lcm4(int b) {
    int a = 4, x = b;
    while (x) { const int t = a % x; a = x; x = t; }
    return 4 / a * b;
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

// Unit width, ring depth and shared memory for a geometry; false if unsupported.
bool plan(const jano_geom& gm, int K, int C, bool literal, AGeo& a) {
    a.K = K; a.C = C; a.F = gm.F; a.H = gm.H; a.W = gm.W;
    a.bf = gm.bf; a.bh = gm.bh; a.bw = gm.bw;
    a.nBh = (gm.H + gm.bh - 1) / gm.bh;
    a.nBw = (gm.W + gm.bw - 1) / gm.bw;
    const int R = gm.bf * gm.bh;
    const int L0 = lcm4(gm.bw);
    const int L = L0 % (4 * kVec) == 0 ? L0 : (4 * kVec) / gcd(L0, 4 * kVec) * L0;   // lcm(L0, 4 kVec)
    if (gm.bh + 1 > 256 || gm.bf > 256 || K + 1 > 256) return false;
    // widest unit (a multiple of L, at most the padded row) whose box fits a
    // TMA box row and whose threads fit a CTA
    const int Wr = (gm.W + L - 1) / L * L;
    int Wc = JANO_ANALYZER_WC > 0 ? JANO_ANALYZER_WC / L * L : Wr;
    if (Wc > Wr) Wc = Wr;
    while (Wc > L && (Wc + 4 > 256 || (long long)R * (Wc / (4 * kVec)) * (K - 1) + 32 > 1024)) Wc -= L;
    if (Wc < L || Wc + 4 > 256 || (long long)R * (Wc / (4 * kVec)) * (K - 1) + 32 > 1024) return false;
    a.Wc = Wc;
    a.LA = Wc + 4;
    a.n_wc = (gm.W + Wc - 1) / Wc;
    a.n_units = ((gm.F + gm.bf - 1) / gm.bf) * a.nBh * a.n_wc;
    a.NP = R * (Wc / (4 * kVec));
    a.NC = (a.NP * (K - 1) + 31) / 32 * 32;
    a.bytesA = a.LA * (gm.bh + 1) * gm.bf * (K + 1) * 4;
    a.bytesB = Wc * gm.bh * (literal ? K + 1 : K - 1) * 4;   // snapshots 0..K or 1..K-1
    a.offB = (a.bytesA + 127) / 128 * 128;
    a.stage_bytes = (a.offB + a.bytesB + 127) / 128 * 128;
    const long long fixed = (long long)(K - 1) * R * Wc * 4 + 128 + 16;   // red + slack + abort
    auto stages_for = [&](long long budget) {
        long long n = (budget - fixed) / (a.stage_bytes + 16);
        return n > kMaxStages ? kMaxStages : n;
    };
    long long budget = JANO_ANALYZER_SMEM_KB * 1024ll;
    if (JANO_ANALYZER_SMEM_KB == 0) {
        budget = 220 * 1024ll;
        for (long long b : {72 * 1024ll, 110 * 1024ll})
            if (stages_for(b) >= 4) { budget = b; break; }
    }
    const long long S = stages_for(budget);
    if (S < 2) return false;
    a.S = (int)S;
    a.red_off = a.S * a.stage_bytes + 16 * a.S + 16;     // barriers and abort flag sit below red
    a.smem = a.red_off + (K - 1) * R * Wc * 4 + 128;
    return true;
}

// Frame-group plan.  Measured on B200 over the video latents of the pages'
// configurations (units of 32 or 64 columns, 2 to 6 frames, rings of 2 or 3
// stages): 32 columns, 3 frames and a 2-stage ring (15 KB stages, 64
// registers a thread, so seven 128-thread CTAs fit an SM) is the fastest;
// wider units or deeper rings leave fewer CTAs per SM and lose more than the
// L2 bytes they save.  A latent with fewer than two such units per SM (the
// image and tiny latents: one frame, or a few small frames) takes units of
// one frame and a 4-stage ring instead, for more units in flight.  The unit
// shape does not change a block's arithmetic (each thread adds its channels
// and steps in the same order, and the shuffle tree is fixed), so every
// shape, and every frame slab of a latent, gives the same bits.
#ifndef JANO_ANALYZER_FG
#define JANO_ANALYZER_FG 1
#endif
#ifndef JANO_ANALYZER_FG_WC
#define JANO_ANALYZER_FG_WC 32
#endif
#ifndef JANO_ANALYZER_FG_G
#define JANO_ANALYZER_FG_G 3
#endif
#ifndef JANO_ANALYZER_FG_S
#define JANO_ANALYZER_FG_S 2
#endif
constexpr int kFgK = 5;
static_assert(JANO_ANALYZER_FG_WC % 32 == 0 && JANO_ANALYZER_FG_WC + 4 <= 256, "unit width");
static_assert(JANO_ANALYZER_FG_S >= 2 && JANO_ANALYZER_FG_S <= kMaxStages && kMaxStages >= 4, "ring depth");

bool fg_eligible(const jano_geom& gm, int K, bool literal) {
    if (!JANO_ANALYZER_FG || literal || K != kFgK || gm.bf != 1) return false;
    if (gm.bh != 1 && gm.bh != 2 && gm.bh != 4) return false;
    return gm.bw >= 1 && gm.bw <= 32 && (gm.bw & (gm.bw - 1)) == 0;
}

bool plan_fg(const jano_geom& gm, int K, int C, bool literal, int sms, FGeo& a) {
    if (!fg_eligible(gm, K, literal)) return false;
    a.C = C; a.F = gm.F; a.H = gm.H; a.W = gm.W;
    a.bh = gm.bh; a.bw = gm.bw;
    a.nBh = (gm.H + gm.bh - 1) / gm.bh;
    a.nBw = (gm.W + gm.bw - 1) / gm.bw;
    a.Wc = JANO_ANALYZER_FG_WC;
    a.G = std::min(JANO_ANALYZER_FG_G, gm.F);
    a.S = JANO_ANALYZER_FG_S;
    a.LA = a.Wc + 4;
    a.n_wc = (gm.W + a.Wc - 1) / a.Wc;
    a.n_rg = (gm.H + 3) / 4;
    long long n_units = (long long)((gm.F + a.G - 1) / a.G) * a.n_rg * a.n_wc;
    if (n_units < 2ll * sms && a.G > 1) {
        a.G = 1;
        a.S = 4;
        n_units = (long long)gm.F * a.n_rg * a.n_wc;
    }
    if (n_units > (1ll << 30)) return false;
    a.n_units = (int)n_units;
    a.n_warps = a.G * a.Wc / 32;
    if ((a.n_warps + 1) * 32 > kFgMaxThreads) return false;
    a.bytesA = a.LA * 5 * a.G * (K + 1) * 4;
    a.bytesB = a.Wc * 4 * (K - 1) * 4;
    a.offB = (a.bytesA + 127) / 128 * 128;
    a.stage_bytes = (a.offB + a.bytesB + 127) / 128 * 128;
    a.smem = a.S * a.stage_bytes + 16 * a.S + 16 + 128;
    return a.smem <= 220 * 1024;
}

}  // namespace

bool analyzer_supported(const jano_geom& g, int K, int C, bool literal) {
    AGeo a;
    FGeo b;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return plan_fg(g, K, C, literal, sms, b) || plan(g, K, C, literal, a);
}

namespace {
cudaError_t launch_fg(const float* lat, int K, int C, const jano_geom& gm, float w_t, float w_s,
                      float* scores, int* err, cudaStream_t st, bool& taken) {
    taken = false;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    FGeo a;
    if (!plan_fg(gm, K, C, false, sms, a)) return cudaSuccess;
    taken = true;
    a.w_t = w_t;
    a.w_s = w_s;
    auto fn = encode_fn();
    if (!fn) return cudaErrorInvalidValue;
    const cuuint64_t dims[5] = {(cuuint64_t)gm.W, (cuuint64_t)gm.H, (cuuint64_t)gm.F, (cuuint64_t)C,
                                (cuuint64_t)(K + 1)};
    const cuuint64_t strides[4] = {(cuuint64_t)gm.W * 4, (cuuint64_t)gm.H * gm.W * 4,
                                   (cuuint64_t)gm.F * gm.H * gm.W * 4,
                                   (cuuint64_t)C * gm.F * gm.H * gm.W * 4};
    const cuuint32_t boxA[5] = {(cuuint32_t)a.LA, 5, (cuuint32_t)a.G, 1, (cuuint32_t)K + 1};
    const cuuint32_t boxB[5] = {(cuuint32_t)a.Wc, 4, 1, 1, (cuuint32_t)(K - 1)};
    const cuuint32_t es[5] = {1, 1, 1, 1, 1};
    CUtensorMap mA, mB;
    if (fn(&mA, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 5, const_cast<float*>(lat), dims, strides, boxA, es,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
        fn(&mB, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 5, const_cast<float*>(lat), dims, strides, boxB, es,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    static DeviceOnce opted_in;
    if (!opted_in.done(dev)) {
        cudaError_t e = cudaFuncSetAttribute(analyzer_fg_kernel<kFgK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             224 * 1024);
        if (e != cudaSuccess) return e;
        opted_in.mark(dev);
    }
    const int threads = (a.n_warps + 1) * 32;
    // resident CTAs per SM, asked once per device and unit shape
    static std::atomic<int> occupancy[64][JANO_ANALYZER_FG_G + 1][kMaxStages + 1];   // by G and S
    int per = dev < 64 ? occupancy[dev][a.G][a.S].load(std::memory_order_relaxed) : 0;
    if (per < 1) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, analyzer_fg_kernel<kFgK>, threads,
                                                          (size_t)a.smem) != cudaSuccess || per < 1)
            per = 1;
        if (dev < 64) occupancy[dev][a.G][a.S].store(per, std::memory_order_relaxed);
    }
    const int grid = a.n_units < per * sms ? a.n_units : per * sms;
    analyzer_fg_kernel<kFgK><<<grid, threads, (size_t)a.smem, st>>>(mA, mB, a, scores, err);
    return cudaGetLastError();
}
}  // namespace

cudaError_t launch_block_scores(const float* lat, int K, int C, const jano_geom& gm,
                                float w_t, float w_s, bool literal, float* scores, int* err,
                                cudaStream_t st) {
    if (!literal) {
        bool taken = false;
        const cudaError_t e = launch_fg(lat, K, C, gm, w_t, w_s, scores, err, st, taken);
        if (taken) return e;
    }
    AGeo a;
    if (!plan(gm, K, C, literal, a)) return cudaErrorInvalidValue;
    a.w_t = w_t;
    a.w_s = w_s;
    auto fn = encode_fn();
    if (!fn) return cudaErrorInvalidValue;
    const cuuint64_t dims[5] = {(cuuint64_t)gm.W, (cuuint64_t)gm.H, (cuuint64_t)gm.F, (cuuint64_t)C,
                                (cuuint64_t)(K + 1)};
    const cuuint64_t strides[4] = {(cuuint64_t)gm.W * 4, (cuuint64_t)gm.H * gm.W * 4,
                                   (cuuint64_t)gm.F * gm.H * gm.W * 4,
                                   (cuuint64_t)C * gm.F * gm.H * gm.W * 4};
    const cuuint32_t boxA[5] = {(cuuint32_t)a.Wc + 4, (cuuint32_t)gm.bh + 1, (cuuint32_t)gm.bf, 1,
                                (cuuint32_t)K + 1};
    const cuuint32_t boxB[5] = {(cuuint32_t)a.Wc, (cuuint32_t)gm.bh, 1, 1,
                                (cuuint32_t)(literal ? K + 1 : K - 1)};
    const cuuint32_t es[5] = {1, 1, 1, 1, 1};
    CUtensorMap mA, mB;
    if (fn(&mA, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 5, const_cast<float*>(lat), dims, strides, boxA, es,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
        fn(&mB, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 5, const_cast<float*>(lat), dims, strides, boxB, es,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;

    const size_t smem = (size_t)a.smem;
    static DeviceOnce opted_in[2];   // per-device shared-memory opt-in, per instantiation
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (!opted_in[literal].done(dev)) {
        cudaError_t e = cudaFuncSetAttribute(literal ? analyzer_kernel<true> : analyzer_kernel<false>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, 224 * 1024);
        if (e != cudaSuccess) return e;
        opted_in[literal].mark(dev);
    }
    const int threads = a.NC + 32;
    // resident CTAs per SM: shared memory (228 KB, 1 KB reserved per CTA) and threads
    int per_sm = (228 * 1024) / (a.smem + 1024);
    if (per_sm > 2048 / threads) per_sm = 2048 / threads;
    if (per_sm < 1) per_sm = 1;
    const int grid = a.n_units < per_sm * sms ? a.n_units : per_sm * sms;
    if (literal) analyzer_kernel<true><<<grid, threads, smem, st>>>(mA, mB, a, scores, err);
    else analyzer_kernel<false><<<grid, threads, smem, st>>>(mA, mB, a, scores, err);
    return cudaGetLastError();
}

}  // namespace jano
