// spectral.cu -- frequency-domain block complexity, the FFT baseline the
// analyzer is compared with (Jano pages: zh technical summary 1 and 2.1,
// where a complexity measure taken from the FFT of the early, noise-dominated
// latent predicts convergence far worse than the gradient score; fr technical
// summary 2.A).  The pages give no formula for it; this is its plainest form:
//
//   S_b = 1/C sum_c 1/n_b^2 sum_{u in U_hi} |X_{c,b}(u)|^2
//
// with X_{c,b} the 3-D DFT of block b of channel c over the block's own
// elements (n_b = m_f m_h m_w of them; edge blocks are smaller, as the
// analyzer's are), and U_hi the frequencies whose folded index
// min(u, m - u) reaches `cutoff` on at least one axis.  By Parseval's
// theorem cutoff 0 gives the mean square of the block, and cutoff 1 its
// variance (everything but the DC bin).
//
// One thread per (block, channel group), 32 neighbouring blocks per warp so
// that each block row is one coalesced 16-byte copy per thread.  A thread
// copies several channels of its block into shared memory at once, then
// transforms them one by one in registers: radix-2 FFTs along w, h and f
// (lengths 1, 2, 4, 8, whose twiddles are the eighth roots of unity, applied
// as sign swaps where exact), also for edge blocks whose extents divide 8.
// Other lengths take the DFT by its definition.  The per-channel energies are
// summed in a fixed order (deterministic).  HBM bound: one snapshot is read
// once (19.4 MB for the large video latent) and one float per block written.
#include "jano_common.cuh"

namespace jano {
namespace {

constexpr int kLanes = 32;     // blocks per CTA (adjacent along w)
constexpr int kGroups = 4;     // channel groups per CTA
constexpr float kHalfSqrt2 = 0.70710678118654752440f;

__device__ __forceinline__ constexpr int fold(int u, int m) { return u < m - u ? u : m - u; }
__device__ __forceinline__ bool divides8(int m) { return m == 1 || m == 2 || m == 4 || m == 8; }

__device__ __forceinline__ constexpr int bit_reverse(int i, int n) {
    int r = 0;
    for (int b = 1; b < n; b <<= 1) r = (r << 1) | ((i & b) ? 1 : 0);
    return r;
}

// x *= exp(-2 pi i e / 8) for an integer e known at compile time after
// unrolling: exact sign swaps for multiples of a quarter turn.
__device__ __forceinline__ void rotate_eighths(float& xr, float& xi, int e) {
    e &= 7;
    if (e == 0) return;
    if (e == 2) { const float t = xr; xr = xi; xi = -t; return; }
    if (e == 4) { xr = -xr; xi = -xi; return; }
    if (e == 6) { const float t = xr; xr = -xi; xi = t; return; }
    const float c = (e == 1 || e == 7) ? kHalfSqrt2 : -kHalfSqrt2;   // cos(2 pi e / 8)
    const float s = (e == 1 || e == 3) ? kHalfSqrt2 : -kHalfSqrt2;   // sin(2 pi e / 8)
    const float nr = fmaf(xr, c, xi * s);
    const float ni = fmaf(xi, c, -(xr * s));
    xr = nr;
    xi = ni;
}

// In-place forward DFT of length N (1, 2, 4 or 8) of the complex sequence
// (re[k*S], im[k*S]), k = 0..N-1: radix-2 decimation in frequency, so the
// input is taken in natural order and frequency u lands in slot
// bit_reverse(u) (every index a compile-time constant after unrolling).
template <int N, int S>
__device__ __forceinline__ void fft_small(float* re, float* im) {
#pragma unroll
    for (int len = N; len >= 2; len >>= 1)
#pragma unroll
        for (int i = 0; i < N; i += len)
#pragma unroll
            for (int k = 0; k < len / 2; ++k) {
                const int a = (i + k) * S, b = (i + k + len / 2) * S;
                const float ar = re[a], ai = im[a];
                float dr = ar - re[b], di = ai - im[b];
                re[a] = ar + re[b];
                im[a] = ai + im[b];
                rotate_eighths(dr, di, k * (8 / len));
                re[b] = dr;
                im[b] = di;
            }
}

// Length m (a divisor of 8, at most B) along an axis of B slots, stride S.
template <int B, int S>
__device__ __forceinline__ void fft_runtime(float* re, float* im, int m) {
    if (m == B) { fft_small<B, S>(re, im); return; }
    if constexpr (B >= 8) { if (m == 4) { fft_small<4, S>(re, im); return; } }
    if constexpr (B >= 4) { if (m == 2) { fft_small<2, S>(re, im); return; } }
}

// 16 bytes global -> shared (`bytes` 16 copies, 0 writes zeros), and the
// wait for every copy this thread has issued.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Block of one channel into registers: one 16-byte load per row when the
// row is whole and aligned, else element loads; slots outside the block
// hold 0 and are never counted.
template <int BF, int BH, int BW>
__device__ __forceinline__ void load_block(const float* __restrict__ p, size_t plane, int W, int mf,
                                           int mh, int mw, bool vec4, float (&v)[BF * BH * BW]) {
#pragma unroll
    for (int f = 0; f < BF; ++f)
#pragma unroll
        for (int h = 0; h < BH; ++h) {
            const float* row = p + f * plane + (size_t)h * W;
            const bool in = f < mf && h < mh;
            if constexpr (BW % 4 == 0) {
                if (vec4 && in) {
#pragma unroll
                    for (int w = 0; w < BW; w += 4) {
                        const float4 q = __ldg(reinterpret_cast<const float4*>(row + w));
                        v[(f * BH + h) * BW + w + 0] = q.x;
                        v[(f * BH + h) * BW + w + 1] = q.y;
                        v[(f * BH + h) * BW + w + 2] = q.z;
                        v[(f * BH + h) * BW + w + 3] = q.w;
                    }
                    continue;
                }
            }
#pragma unroll
            for (int w = 0; w < BW; ++w)
                v[(f * BH + h) * BW + w] = (in && w < mw) ? __ldg(row + w) : 0.f;
        }
}

// High-band energy / n^2 of one block held in registers, extents dividing 8
// (kFull: the extents are the block's, known at compile time, so that the
// transform lengths, the bit reversal and the folding all fold away).
template <int BF, int BH, int BW, bool kFull>
__device__ __forceinline__ float block_energy_fft(const float (&v)[BF * BH * BW], int mf_rt, int mh_rt,
                                                  int mw_rt, int cutoff) {
    constexpr int n = BF * BH * BW;
    const int mf = kFull ? BF : mf_rt, mh = kFull ? BH : mh_rt, mw = kFull ? BW : mw_rt;
    float re[n], im[n];
#pragma unroll
    for (int i = 0; i < n; ++i) { re[i] = v[i]; im[i] = 0.f; }
    if constexpr (BW > 1) {
#pragma unroll
        for (int r = 0; r < BF * BH; ++r) fft_runtime<BW, 1>(re + r * BW, im + r * BW, mw);
    }
    if constexpr (BH > 1) {
#pragma unroll
        for (int f = 0; f < BF; ++f)
#pragma unroll
            for (int w = 0; w < BW; ++w)
                fft_runtime<BH, BW>(re + f * BH * BW + w, im + f * BH * BW + w, mh);
    }
    if constexpr (BF > 1) {
#pragma unroll
        for (int hw = 0; hw < BH * BW; ++hw) fft_runtime<BF, BH * BW>(re + hw, im + hw, mf);
    }
    // slot (sf, sh, sw) holds frequency (bit_reverse(sf, mf), ...)
    float e = 0.f;
#pragma unroll
    for (int sf = 0; sf < BF; ++sf)
#pragma unroll
        for (int sh = 0; sh < BH; ++sh)
#pragma unroll
            for (int sw = 0; sw < BW; ++sw) {
                const int i = (sf * BH + sh) * BW + sw;
                const bool inside = sf < mf && sh < mh && sw < mw;
                const int k = max(fold(bit_reverse(sf, mf), mf),
                                  max(fold(bit_reverse(sh, mh), mh), fold(bit_reverse(sw, mw), mw)));
                const float m2 = fmaf(re[i], re[i], im[i] * im[i]);
                e += (inside && k >= cutoff) ? m2 : 0.f;
            }
    const float nb = (float)(mf * mh * mw);
    return e / (nb * nb);
}

// Any extents: the DFT by its definition, phases reduced exactly as integers
// mod n and their sine and cosine computed.
__device__ __forceinline__ float block_energy_direct(const float* __restrict__ p, size_t plane, int W, int mf,
                                     int mh, int mw, int cutoff) {
    const int n = mf * mh * mw;
    float e = 0.f;
    for (int uf = 0; uf < mf; ++uf)
        for (int uh = 0; uh < mh; ++uh)
            for (int uw = 0; uw < mw; ++uw) {
                const int k = max(fold(uf, mf), max(fold(uh, mh), fold(uw, mw)));
                if (k < cutoff) continue;
                float re = 0.f, im = 0.f;
                for (int f = 0; f < mf; ++f)
                    for (int h = 0; h < mh; ++h)
                        for (int w = 0; w < mw; ++w) {
                            // phase / (2 pi) = uf f / mf + uh h / mh + uw w / mw = q / n
                            const int q = (uf * f * mh * mw + uh * h * mf * mw + uw * w * mf * mh) % n;
                            float s, c;
                            sincospif(2.f * (float)q / (float)n, &s, &c);
                            const float v = __ldg(p + f * plane + (size_t)h * W + w);
                            re = fmaf(v, c, re);
                            im = fmaf(-v, s, im);
                        }
                e = fmaf(re, re, fmaf(im, im, e));
            }
    return e / ((float)n * (float)n);
}

// Block coordinates and extents of block b.
struct BlockAt {
    const float* base;   // channel 0, first element
    int mf, mh, mw;
};

__device__ __forceinline__ BlockAt block_at(const float* x, int b, int F, int H, int W, int bf, int bh,
                                            int bw, int nBh, int nBw) {
    const int wb = b % nBw, t = b / nBw;
    const int hb = t % nBh, fb = t / nBh;
    const int f0 = fb * bf, h0 = hb * bh, w0 = wb * bw;
    BlockAt a;
    a.base = x + (size_t)f0 * H * W + (size_t)h0 * W + w0;
    a.mf = min(bf, F - f0);
    a.mh = min(bh, H - h0);
    a.mw = min(bw, W - w0);
    return a;
}

// Channel-group partial sums of a CTA's 32 blocks, summed in a fixed order.
__device__ __forceinline__ void store_scores(float (&part)[kGroups][kLanes], float acc, bool mine, int b,
                                             int C, float* __restrict__ scores) {
    part[threadIdx.y][threadIdx.x] = acc;
    __syncthreads();
    if (threadIdx.y == 0 && mine) {
        float s = part[0][threadIdx.x];
#pragma unroll
        for (int g = 1; g < kGroups; ++g) s += part[g][threadIdx.x];
        scores[b] = s / (float)C;
    }
}

// The blocks of a BF x BH x BW geometry whose extents divide 8 (every block
// unless an edge is 3, 5, 6 or 7 long), by FFT.
//
// Whole, aligned rows (the usual case) are staged through shared memory:
// each thread issues 16-byte cp.async copies for kChunk channels of its block
// at once (64 floats), so that a CTA has 32 KB in flight and an SM several
// CTAs' worth; only then does it wait and transform them.  A thread reads
// back only what it copied itself, so no barrier is needed.  The staging
// buffer interleaves threads at 16-byte granularity (slot q of thread t at
// stage[q][t]), which keeps the read-back free of bank conflicts.  Other
// blocks (partial rows along w, unaligned rows) load through registers with
// the next channel's block in flight during the current transform.
template <int BF, int BH, int BW>
__global__ void __launch_bounds__(kLanes * kGroups, BF * BH * BW <= 16 ? 5 : 1)
fft_scores_kernel(const float* __restrict__ x, int C, int F, int H, int W, int nBh, int nBw,
                  int n_blocks, int cutoff, bool vec4, float* __restrict__ scores) {
    constexpr int n = BF * BH * BW;
    constexpr int kStageQ = 16;                          // float4 slots per thread
    constexpr bool kStaged = BW % 4 == 0 && n <= 4 * kStageQ;
    constexpr int kChunk = kStaged ? 4 * kStageQ / n : 1;  // channels per staged round
    __shared__ float part[kGroups][kLanes];
    __shared__ __align__(16) float4 stage[kStaged ? kStageQ : 1][kLanes * kGroups];
    const int tid = threadIdx.y * kLanes + threadIdx.x;
    const int b = blockIdx.x * kLanes + threadIdx.x;
    float acc = 0.f;
    bool mine = false;
    if (b < n_blocks) {
        const BlockAt a = block_at(x, b, F, H, W, BF, BH, BW, nBh, nBw);
        mine = divides8(a.mf) && divides8(a.mh) && divides8(a.mw);
        const size_t plane = (size_t)H * W, chan = (size_t)F * plane;
        const bool v4 = vec4 && a.mw == BW;
        const bool full = a.mf == BF && a.mh == BH && a.mw == BW;
        if (mine && kStaged && v4) {
            if constexpr (kStaged) {
                for (int c0 = threadIdx.y; c0 < C; c0 += kGroups * kChunk) {
#pragma unroll
                    for (int j = 0; j < kChunk; ++j) {
                        const int c = c0 + j * kGroups;
                        if (c >= C) break;
#pragma unroll
                        for (int f = 0; f < BF; ++f)
#pragma unroll
                            for (int h = 0; h < BH; ++h) {
                                const bool in = f < a.mf && h < a.mh;
                                const float* row = in ? a.base + c * chan + f * plane + (size_t)h * W : a.base;
#pragma unroll
                                for (int q = 0; q < BW / 4; ++q)
                                    cp_async16(ptx::smem_u32(&stage[j * (n / 4) + (f * BH + h) * (BW / 4) + q][tid]),
                                               row + 4 * q, in ? 16u : 0u);
                            }
                    }
                    cp_async_wait_all();
#pragma unroll
                    for (int j = 0; j < kChunk; ++j) {
                        const int c = c0 + j * kGroups;
                        if (c >= C) break;
                        float v[n];
#pragma unroll
                        for (int q = 0; q < n / 4; ++q) {
                            const float4 t = stage[j * (n / 4) + q][tid];
                            v[4 * q + 0] = t.x;
                            v[4 * q + 1] = t.y;
                            v[4 * q + 2] = t.z;
                            v[4 * q + 3] = t.w;
                        }
                        acc += full ? block_energy_fft<BF, BH, BW, true>(v, a.mf, a.mh, a.mw, cutoff)
                                    : block_energy_fft<BF, BH, BW, false>(v, a.mf, a.mh, a.mw, cutoff);
                    }
                }
            }
        } else if (mine) {
            constexpr bool kPrefetch = n <= 32;    // registers for two blocks and the transform
            float cur[n], nxt[n];
            int c = threadIdx.y;
            if (c < C) load_block<BF, BH, BW>(a.base + c * chan, plane, W, a.mf, a.mh, a.mw, v4, cur);
            for (; c < C; c += kGroups) {
                const bool more = c + kGroups < C;
                if (kPrefetch && more)
                    load_block<BF, BH, BW>(a.base + (c + kGroups) * chan, plane, W, a.mf, a.mh, a.mw, v4, nxt);
                acc += full ? block_energy_fft<BF, BH, BW, true>(cur, a.mf, a.mh, a.mw, cutoff)
                            : block_energy_fft<BF, BH, BW, false>(cur, a.mf, a.mh, a.mw, cutoff);
                if (more) {
                    if constexpr (kPrefetch) {
#pragma unroll
                        for (int i = 0; i < n; ++i) cur[i] = nxt[i];
                    } else {
                        load_block<BF, BH, BW>(a.base + (c + kGroups) * chan, plane, W, a.mf, a.mh, a.mw,
                                               v4, cur);
                    }
                }
            }
        }
    }
    store_scores(part, acc, mine, b, C, scores);
}

// Blocks by the definition: all of them, or (skip_eighths) only those whose
// extents do not all divide 8, which fft_scores_kernel leaves.
__global__ void __launch_bounds__(kLanes * kGroups)
dft_scores_kernel(const float* __restrict__ x, int C, int F, int H, int W, int bf, int bh, int bw,
                  int nBh, int nBw, int n_blocks, int cutoff, bool skip_eighths,
                  float* __restrict__ scores) {
    __shared__ float part[kGroups][kLanes];
    const int b = blockIdx.x * kLanes + threadIdx.x;
    float acc = 0.f;
    bool mine = false;
    if (b < n_blocks) {
        const BlockAt a = block_at(x, b, F, H, W, bf, bh, bw, nBh, nBw);
        mine = !(skip_eighths && divides8(a.mf) && divides8(a.mh) && divides8(a.mw));
        if (mine) {
            const size_t plane = (size_t)H * W, chan = (size_t)F * plane;
            for (int c = threadIdx.y; c < C; c += kGroups)
                acc += block_energy_direct(a.base + c * chan, plane, W, a.mf, a.mh, a.mw, cutoff);
        }
    }
    store_scores(part, acc, mine, b, C, scores);
}

}  // namespace

bool fft_scores_supported(const jano_geom& g) {
    return (long long)g.bf * g.bh * g.bw <= 256;
}

cudaError_t launch_fft_scores(const float* x, int C, const jano_geom& g, int cutoff, float* scores,
                              cudaStream_t st) {
    const int nBf = (g.F + g.bf - 1) / g.bf, nBh = (g.H + g.bh - 1) / g.bh,
              nBw = (g.W + g.bw - 1) / g.bw;
    const int n = nBf * nBh * nBw;
    const dim3 block(kLanes, kGroups);
    const dim3 grid((n + kLanes - 1) / kLanes);
    // rows of 4 along w load as one float4 when every row start is 16-byte aligned
    const bool vec4 = (reinterpret_cast<uintptr_t>(x) & 15) == 0 && g.W % 4 == 0 && g.bw % 4 == 0;
    auto shape = [&](int f, int h, int w) { return g.bf == f && g.bh == h && g.bw == w; };
    auto div8 = [](int m) { return m == 1 || m == 2 || m == 4 || m == 8; };
    bool fft = true;
#define JANO_FFT_LAUNCH(F_, H_, W_) \
    fft_scores_kernel<F_, H_, W_><<<grid, block, 0, st>>>(x, C, g.F, g.H, g.W, nBh, nBw, n, cutoff, vec4, scores)
    if (shape(1, 4, 4)) JANO_FFT_LAUNCH(1, 4, 4);
    else if (shape(1, 2, 2)) JANO_FFT_LAUNCH(1, 2, 2);
    else if (shape(1, 8, 8)) JANO_FFT_LAUNCH(1, 8, 8);
    else if (shape(2, 2, 2)) JANO_FFT_LAUNCH(2, 2, 2);
    else if (shape(2, 4, 4)) JANO_FFT_LAUNCH(2, 4, 4);
    else fft = false;
#undef JANO_FFT_LAUNCH
    // edge extents (the remainders) that do not divide 8 need the direct DFT
    const bool odd_edges = !div8(g.F % g.bf ? g.F % g.bf : g.bf) || !div8(g.H % g.bh ? g.H % g.bh : g.bh) ||
                           !div8(g.W % g.bw ? g.W % g.bw : g.bw);
    if (!fft || odd_edges)
        dft_scores_kernel<<<grid, block, 0, st>>>(x, C, g.F, g.H, g.W, g.bf, g.bh, g.bw, nBh, nBw, n, cutoff,
                                                  fft, scores);
    return cudaGetLastError();
}

}  // namespace jano
