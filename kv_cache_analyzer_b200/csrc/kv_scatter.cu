// kv_scatter.cu -- fused KV-cache update: k_cache[idx[i]] = k_act[i] and
// v_cache[idx[i]] = v_act[i] in one pass (Jano pages: nl technical summary,
// Methodologie 2 "KV Cache Mechanisme"; zh 2.2 item 3).
//
// Pure HBM streaming: every byte of k_act/v_act is read once and written once
// (4 * n_act * heads * d * 2 bytes).  One warp owns one row at a time; its
// lanes move the row's 16-byte vectors with UNROLL independent K and V loads
// in flight per lane before the stores.  Rows are grid-strided over a grid
// sized to fill every SM.  No scratch memory.
//
// Index contract: idx strictly ascending (what the schedule emits).  A row
// whose id is out of range, or not above the previous row's id (a duplicate
// or a step back), raises JANO_EINDEX and is skipped, so an adjacent
// duplicate never races; the extra load hits the line the warp just read.
#include "jano_common.cuh"

namespace jano {
namespace {

constexpr int kWarps = 8;
constexpr int kUnroll = 4;

__global__ void __launch_bounds__(kWarps * 32)
kv_scatter_kernel(const uint4* __restrict__ k_act, const uint4* __restrict__ v_act,
                  const int32_t* __restrict__ idx, int n_act, int row_vec,
                  uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                  int n_tokens, int* err) {
    const int lane = threadIdx.x & 31;
    const int warp = blockIdx.x * kWarps + (threadIdx.x >> 5);
    const int nwarps = gridDim.x * kWarps;
    for (int i = warp; i < n_act; i += nwarps) {
        const int t = __ldg(idx + i);
        if (t < 0 || t >= n_tokens || (i > 0 && __ldg(idx + i - 1) >= t)) {
            if (lane == 0) raise_error(err, JANO_EINDEX);
            continue;
        }
        const uint4* ks = k_act + (size_t)i * row_vec;
        const uint4* vs = v_act + (size_t)i * row_vec;
        uint4* kd = k_cache + (size_t)t * row_vec;
        uint4* vd = v_cache + (size_t)t * row_vec;
        int e = lane;
        for (; e + 32 * (kUnroll - 1) < row_vec; e += 32 * kUnroll) {
            uint4 a[kUnroll], b[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                a[u] = __ldcs(ks + e + 32 * u);
                b[u] = __ldcs(vs + e + 32 * u);
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                __stcs(kd + e + 32 * u, a[u]);
                __stcs(vd + e + 32 * u, b[u]);
            }
        }
        for (; e < row_vec; e += 32) {
            const uint4 a = __ldcs(ks + e);
            const uint4 b = __ldcs(vs + e);
            __stcs(kd + e, a);
            __stcs(vd + e, b);
        }
    }
}

}  // namespace

cudaError_t launch_kv_scatter(const void* k_act, const void* v_act, const int32_t* idx,
                              int n_act, int row_bytes, void* k_cache, void* v_cache,
                              int n_tokens, int* err, cudaStream_t st) {
    if (n_act <= 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int want = (n_act + kWarps - 1) / kWarps;
    const int grid = want < sms * 8 ? want : sms * 8;
    kv_scatter_kernel<<<grid, kWarps * 32, 0, st>>>(
        static_cast<const uint4*>(k_act), static_cast<const uint4*>(v_act), idx, n_act,
        row_bytes / 16, static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache),
        n_tokens, err);
    return cudaGetLastError();
}

}  // namespace jano
