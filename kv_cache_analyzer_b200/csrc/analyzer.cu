// analyzer.cu -- block-wise complexity analyzer (Jano pages: zh technical
// summary 2.1; nl technical summary, Methodologie 1 "Implementatie"; pt 2.A).
//
//   S_b = mean over k=1..K-1, c, (f,h,w) in b of
//         |x_{k+1} - 2x_k + x_{k-1}| + w_t |D_f x_k| + w_s sqrt(D_h x_k^2 + D_w x_k^2)
//
// HBM-bound streaming stencil.  A CTA owns one frame-block x one block-row x
// a width chunk (a whole number of blocks) and every channel.  Thread
// (cg, r, w4) owns four consecutive latent elements of one (f,h) row and the
// channels c = cg, cg+CG, ...; for each channel it walks the K+1 snapshots
// with float4 loads, keeping the (k-1, k, k+1) window in registers.  The
// f+1 / h+1 neighbours of snapshot k are float4 loads that hit L1/L2 (the
// neighbouring rows and frames are being streamed by this and adjacent
// CTAs), the w+1 neighbour of the fourth element is one scalar load.  Per
// element sums go to shared memory and one thread per block adds them in a
// fixed order, so scores are deterministic (no atomics).
#include "jano_common.cuh"

namespace jano {
namespace {

struct AGeo {
    int K, C, F, H, W;
    int bf, bh, bw;
    int nBh, nBw;
    int wchunk;       // latent columns per CTA, multiple of 4 and of bw
    int cg;           // channel groups per CTA
    float w_t, w_s;
};

__device__ __forceinline__ float term(float d2, float df, float dh, float dw, float w_t, float w_s) {
    return fabsf(d2) + w_t * fabsf(df) + w_s * sqrtf(dh * dh + dw * dw);
}

__global__ void __launch_bounds__(1024)
analyzer_kernel(const float* __restrict__ lat, AGeo g, float* __restrict__ scores) {
    extern __shared__ float red[];   // [cg][R][wchunk]
    const int R = g.bf * g.bh;
    const int W4c = g.wchunk >> 2;
    const int tid = threadIdx.x;
    const int w4 = tid % W4c;
    const int r = (tid / W4c) % R;
    const int cg = tid / (W4c * R);

    const int fb = blockIdx.z, hb = blockIdx.y;
    const int f0 = fb * g.bf, h0 = hb * g.bh, w0 = blockIdx.x * g.wchunk;
    const int rows_f = min(g.bf, g.F - f0), rows_h = min(g.bh, g.H - h0);
    const int fr = r / g.bh, hr = r % g.bh;
    const int f = f0 + fr, h = h0 + hr, w = w0 + 4 * w4;

    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    if (fr < rows_f && hr < rows_h && w < g.W) {
        const size_t plane = (size_t)g.H * g.W;
        const size_t snap = (size_t)g.C * g.F * plane;
        const bool has_f = f + 1 < g.F, has_h = h + 1 < g.H, has_w = w + 4 < g.W;
        for (int c = cg; c < g.C; c += g.cg) {
            const float* p = lat + ((size_t)c * g.F + f) * plane + (size_t)h * g.W + w;
            float4 xm = __ldg(reinterpret_cast<const float4*>(p));
            float4 x0 = __ldg(reinterpret_cast<const float4*>(p + snap));
            for (int k = 1; k < g.K; ++k) {
                const float* pk = p + (size_t)k * snap;
                const float4 xp = __ldg(reinterpret_cast<const float4*>(pk + snap));
                const float4 nf = has_f ? __ldg(reinterpret_cast<const float4*>(pk + plane)) : x0;
                const float4 nh = has_h ? __ldg(reinterpret_cast<const float4*>(pk + g.W)) : x0;
                const float nw = has_w ? __ldg(pk + 4) : x0.w;
                a0 += term(xp.x - 2.f * x0.x + xm.x, nf.x - x0.x, nh.x - x0.x, x0.y - x0.x, g.w_t, g.w_s);
                a1 += term(xp.y - 2.f * x0.y + xm.y, nf.y - x0.y, nh.y - x0.y, x0.z - x0.y, g.w_t, g.w_s);
                a2 += term(xp.z - 2.f * x0.z + xm.z, nf.z - x0.z, nh.z - x0.z, x0.w - x0.z, g.w_t, g.w_s);
                a3 += term(xp.w - 2.f * x0.w + xm.w, nf.w - x0.w, nh.w - x0.w, nw - x0.w, g.w_t, g.w_s);
                xm = x0;
                x0 = xp;
            }
        }
    }
    float* dst = red + ((size_t)cg * R + r) * g.wchunk + 4 * w4;
    dst[0] = a0; dst[1] = a1; dst[2] = a2; dst[3] = a3;
    __syncthreads();

    const int nb = g.wchunk / g.bw;
    for (int ob = tid; ob < nb; ob += blockDim.x) {
        const int ws = w0 + ob * g.bw;
        if (ws >= g.W) continue;
        const int cols = min(g.bw, g.W - ws);
        float s = 0.f;
        for (int q = 0; q < g.cg; ++q)
            for (int rr = 0; rr < R; ++rr) {
                const float* src = red + ((size_t)q * R + rr) * g.wchunk + ob * g.bw;
                for (int e = 0; e < g.bw; ++e) s += src[e];
            }
        const float cnt = (float)(g.K - 1) * (float)g.C * (float)(rows_f * rows_h * cols);
        scores[((size_t)fb * g.nBh + hb) * g.nBw + (ws / g.bw)] = s / cnt;
    }
}

int lcm4(int b) {
    int a = 4, x = b;
    while (x) { const int t = a % x; a = x; x = t; }
    return 4 / a * b;
}

}  // namespace

cudaError_t launch_block_scores(const float* lat, int K, int C, const jano_geom& g,
                                float w_t, float w_s, float* scores, int* err,
                                cudaStream_t st) {
    (void)err;
    AGeo a;
    a.K = K; a.C = C; a.F = g.F; a.H = g.H; a.W = g.W;
    a.bf = g.bf; a.bh = g.bh; a.bw = g.bw;
    a.nBh = (g.H + g.bh - 1) / g.bh;
    a.nBw = (g.W + g.bw - 1) / g.bw;
    a.w_t = w_t; a.w_s = w_s;
    const int R = g.bf * g.bh;
    const int L = lcm4(g.bw);
    // width chunk: the whole row when it fits, else the widest multiple of L
    // that keeps R * chunk/4 <= 256 threads per channel group
    int wchunk = ((g.W + L - 1) / L) * L;
    while (R * (wchunk / 4) > 256 && wchunk > L) wchunk = ((wchunk / 2 + L - 1) / L) * L;
    a.wchunk = wchunk;
    const int per_cg = R * (wchunk / 4);
    int cg = 512 / per_cg;
    if (cg < 1) cg = 1;
    if (cg > C) cg = C;
    a.cg = cg;
    const int threads = cg * per_cg;
    const size_t smem = sizeof(float) * (size_t)cg * R * wchunk;
    const dim3 grid((g.W + wchunk - 1) / wchunk, a.nBh, (g.F + g.bf - 1) / g.bf);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(analyzer_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    analyzer_kernel<<<grid, threads, smem, st>>>(lat, a, scores);
    return cudaGetLastError();
}

// Largest block footprint the analyzer launch supports (one channel group).
bool analyzer_supported(const jano_geom& g) {
    const int R = g.bf * g.bh;
    const int L = lcm4(g.bw);
    return R * (L / 4) <= 1024 && (size_t)R * L * sizeof(float) <= 200 * 1024;
}

}  // namespace jano
