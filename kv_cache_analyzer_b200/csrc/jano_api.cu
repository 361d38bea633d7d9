// jano_api.cu -- the exported C ABI of libjano: argument validation on the
// host, then one or more asynchronous launches on the caller's stream.  See
// include/jano.h for the contract of each entry point.
#include <cmath>
#include <cstdint>
#include <climits>

#include "jano_common.cuh"

namespace jano {

__device__ int g_device_error = JANO_OK;

int* device_error_word() {
    // cached per device; several host threads may fill a slot, all with the
    // same address
    static std::atomic<int*> addr[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    int* a = addr[dev].load(std::memory_order_acquire);
    if (!a) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
        a = static_cast<int*>(p);
        addr[dev].store(a, std::memory_order_release);
    }
    return a;
}

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

jano_status from_cuda(cudaError_t e) { return e == cudaSuccess ? JANO_OK : JANO_ECUDA; }

jano_status check_geom(const jano_geom* g, bool need_patch) {
    if (!g) return JANO_EINVAL;
    if (g->F < 1 || g->H < 1 || g->W < 1 || g->bf < 1 || g->bh < 1 || g->bw < 1)
        return JANO_EINVAL;
    if (need_patch) {
        if (g->pf < 1 || g->ph < 1 || g->pw < 1) return JANO_EINVAL;
        if (g->F % g->pf || g->H % g->ph || g->W % g->pw) return JANO_ESHAPE;
        const long long nt = (long long)(g->F / g->pf) * (g->H / g->ph) * (g->W / g->pw);
        if (nt > INT_MAX) return JANO_EUNSUPPORTED;
    }
    const long long nb = (long long)((g->F + g->bf - 1) / g->bf) * ((g->H + g->bh - 1) / g->bh) *
                         ((g->W + g->bw - 1) / g->bw);
    if (nb > INT_MAX) return JANO_EUNSUPPORTED;
    return JANO_OK;
}

}  // namespace
}  // namespace jano

using namespace jano;

extern "C" {

namespace {
jano_status block_scores_impl(const float* lat, int K, int C, const jano_geom* g, float w_temporal,
                              float w_spatial, bool literal, float* scores, void* stream) {
    if (!lat || !scores) return JANO_EINVAL;
    if (K < 2 || C < 1) return JANO_EINVAL;
    if (!std::isfinite(w_temporal) || !std::isfinite(w_spatial)) return JANO_EINVAL;
    const jano_status gs = check_geom(g, false);
    if (gs != JANO_OK) return gs;
    if (g->W % 4) return JANO_EUNSUPPORTED;
    if (!aligned16(lat)) return JANO_EALIGN;
    if (!analyzer_supported(*g, K, C, literal)) return JANO_EUNSUPPORTED;
    int* err = device_error_word();
    if (!err) return JANO_ECUDA;
    return from_cuda(launch_block_scores(lat, K, C, *g, w_temporal, w_spatial, literal, scores, err,
                                         static_cast<cudaStream_t>(stream)));
}
}  // namespace

jano_status jano_block_scores(const float* lat, int K, int C, const jano_geom* g,
                              float w_temporal, float w_spatial, float* scores,
                              void* stream) {
    return block_scores_impl(lat, K, C, g, w_temporal, w_spatial, false, scores, stream);
}

jano_status jano_block_scores_literal(const float* lat, int K, int C, const jano_geom* g,
                                      float w_temporal, float w_spatial, float* scores,
                                      void* stream) {
    return block_scores_impl(lat, K, C, g, w_temporal, w_spatial, true, scores, stream);
}

jano_status jano_classify(const float* scores, int n_blocks, float frac_active,
                          float frac_static, uint8_t* levels, void* stream) {
    if (!scores || !levels || n_blocks < 1) return JANO_EINVAL;
    if (!(frac_active >= 0.0f && frac_active <= 1.0f) || !(frac_static >= 0.0f && frac_static <= 1.0f))
        return JANO_EINVAL;
    const long long bpA = std::llround((double)frac_active * 10000.0);
    const long long bpS = std::llround((double)frac_static * 10000.0);
    if (bpA + bpS > 10000) return JANO_EINVAL;
    const long long nA = bpA * n_blocks / 10000;
    const long long nS = bpS * n_blocks / 10000;
    int* err = device_error_word();
    if (!err) return JANO_ECUDA;
    return from_cuda(launch_classify(scores, n_blocks, nS, (long long)n_blocks - nA, levels, err,
                                     static_cast<cudaStream_t>(stream)));
}

size_t jano_build_schedule_workspace_bytes(const jano_geom* g) {
    if (check_geom(g, true) != JANO_OK) return 0;
    return schedule_workspace_bytes(*g);
}

jano_status jano_build_schedule(const uint8_t* block_levels, const jano_geom* g,
                                const jano_sched_cfg* c, int32_t* offsets, int32_t* idx,
                                size_t idx_capacity, uint8_t* token_levels, void* workspace,
                                size_t ws_bytes, void* stream) {
    if (!block_levels || !c || !offsets || !idx || !workspace) return JANO_EINVAL;
    const jano_status gs = check_geom(g, true);
    if (gs != JANO_OK) return gs;
    if (c->T < 1 || c->warmup < 0 || c->cooldown < 0 || c->warmup + c->cooldown > c->T ||
        c->period_moderate < 1 || c->period_static < 1)
        return JANO_EINVAL;
    if (c->T > 65535) return JANO_EUNSUPPORTED;
    const long long nt = (long long)(g->F / g->pf) * (g->H / g->ph) * (g->W / g->pw);
    if (nt * c->T > INT_MAX) return JANO_EUNSUPPORTED;
    if (idx_capacity < (size_t)(nt * c->T)) return JANO_EINVAL;
    if (ws_bytes < schedule_workspace_bytes(*g)) return JANO_EINVAL;
    if (!aligned16(workspace)) return JANO_EALIGN;
    int* err = device_error_word();
    if (!err) return JANO_ECUDA;
    return from_cuda(launch_build_schedule(block_levels, *g, *c, offsets, idx, token_levels,
                                           workspace, err, static_cast<cudaStream_t>(stream)));
}

jano_status jano_kv_scatter(const void* k_act, const void* v_act, const int32_t* idx, int n_act,
                            int heads, int d, void* k_cache, void* v_cache, int n_tokens,
                            void* stream) {
    if (n_act < 0 || heads < 1 || d < 1 || n_tokens < 1) return JANO_EINVAL;
    if (n_act == 0) return JANO_OK;
    if (!k_act || !v_act || !idx || !k_cache || !v_cache) return JANO_EINVAL;
    const long long row_bytes = (long long)heads * d * 2;
    if (row_bytes % 16) return JANO_EUNSUPPORTED;
    if (row_bytes > INT_MAX) return JANO_EUNSUPPORTED;
    if (!aligned16(k_act) || !aligned16(v_act) || !aligned16(k_cache) || !aligned16(v_cache))
        return JANO_EALIGN;
    int* err = device_error_word();
    if (!err) return JANO_ECUDA;
    return from_cuda(launch_kv_scatter(k_act, v_act, idx, n_act, (int)row_bytes, k_cache, v_cache,
                                       n_tokens, err, static_cast<cudaStream_t>(stream)));
}

jano_status jano_active_attention(const void* q_act, const void* k_cache, const void* v_cache,
                                  const int32_t* idx, int n_act, int n_tokens, int heads, int d,
                                  float scale, void* out, void* stream) {
    if (n_act < 0 || n_tokens < 1 || heads < 1) return JANO_EINVAL;
    if (!(scale > 0.0f) || !std::isfinite(scale)) return JANO_EINVAL;
    if (d != 64 && d != 128) return JANO_EUNSUPPORTED;
    if (heads > 65535) return JANO_EUNSUPPORTED;
    if (n_act == 0) return JANO_OK;
    if (!q_act || !k_cache || !v_cache || !idx || !out) return JANO_EINVAL;
    if (!aligned16(q_act) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
        return JANO_EALIGN;
    int* err = device_error_word();
    if (!err) return JANO_ECUDA;
    return from_cuda(launch_active_attention(q_act, k_cache, v_cache, idx, n_act, n_tokens, heads,
                                             d, scale, out, err, static_cast<cudaStream_t>(stream)));
}

jano_status jano_active_attention_split(const void* q_act, const void* k_cache, const void* v_cache,
                                        const int32_t* idx, int n_act, int n_tokens, int heads, int d,
                                        float scale, int n_split, void* workspace, size_t ws_bytes,
                                        void* out, void* stream) {
    if (n_act < 0 || n_tokens < 1 || heads < 1) return JANO_EINVAL;
    if (!(scale > 0.0f) || !std::isfinite(scale)) return JANO_EINVAL;
    if (d != 64 && d != 128) return JANO_EUNSUPPORTED;
    if (heads > 65535) return JANO_EUNSUPPORTED;
    if (n_split < 1 || n_split > attention_key_tiles(n_tokens) || n_split > 65535) return JANO_EINVAL;
    if (n_split == 1)
        return jano_active_attention(q_act, k_cache, v_cache, idx, n_act, n_tokens, heads, d, scale,
                                     out, stream);
    if (n_act == 0) return JANO_OK;
    if (!workspace || ws_bytes < attention_workspace_bytes(n_act, heads, d, n_split)) return JANO_EINVAL;
    if (!aligned16(workspace)) return JANO_EALIGN;
    if (!q_act || !k_cache || !v_cache || !idx || !out) return JANO_EINVAL;
    if (!aligned16(q_act) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
        return JANO_EALIGN;
    int* err = device_error_word();
    if (!err) return JANO_ECUDA;
    return from_cuda(launch_active_attention(q_act, k_cache, v_cache, idx, n_act, n_tokens, heads, d,
                                             scale, out, err, static_cast<cudaStream_t>(stream),
                                             n_split, workspace));
}

size_t jano_active_attention_workspace_bytes(int n_act, int heads, int d, int n_split) {
    if (n_act <= 0 || heads <= 0 || d <= 0 || n_split <= 1) return 0;
    return attention_workspace_bytes(n_act, heads, d, n_split);
}

int jano_active_attention_splits_on(int n_act, int n_tokens, int heads, int d, int sm_count) {
    if (n_act <= 0 || n_tokens < 1 || heads < 1 || (d != 64 && d != 128) || sm_count < 1) return 1;
    return attention_split_count(n_act, n_tokens, heads, sm_count);
}

int jano_active_attention_splits(int n_act, int n_tokens, int heads, int d) {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 1;
    return jano_active_attention_splits_on(n_act, n_tokens, heads, d, sms);
}

jano_status jano_gather_gemm(const void* x, int n_x, const int32_t* gather, int m, const void* w,
                             int n, int k, const int32_t* scatter, void* out, int n_out,
                             void* stream) {
    if (n_x < 1 || m < 0 || n < 1 || k < 1 || n_out < 1) return JANO_EINVAL;
    if (m == 0) return JANO_OK;
    if (!x || !w || !out) return JANO_EINVAL;
    if (!gather && m > n_x) return JANO_ESHAPE;
    if (!scatter && m > n_out) return JANO_ESHAPE;
    if (k % 8 || n % 8) return JANO_EUNSUPPORTED;
    if (!aligned16(x) || !aligned16(w) || !aligned16(out)) return JANO_EALIGN;
    int* err = device_error_word();
    if (!err) return JANO_ECUDA;
    ProjSeg seg{out, scatter, n, n_out};
    return from_cuda(launch_projection(x, n_x, gather, m, w, n, k, 1, &seg, err,
                                       static_cast<cudaStream_t>(stream)));
}

jano_status jano_qkv_project(const void* x, int n_tokens, const int32_t* idx, int n_act,
                             const void* w_qkv, int hd, int k, void* q_act, void* k_cache,
                             void* v_cache, void* stream) {
    if (n_tokens < 1 || n_act < 0 || hd < 1 || k < 1) return JANO_EINVAL;
    if (n_act == 0) return JANO_OK;
    if (!x || !idx || !w_qkv || !q_act || !k_cache || !v_cache) return JANO_EINVAL;
    if (k % 8 || projection_tile_n(3 * hd, hd, 3) == 0) return JANO_EUNSUPPORTED;
    if (3ll * hd > INT_MAX) return JANO_EUNSUPPORTED;
    if (!aligned16(x) || !aligned16(w_qkv) || !aligned16(q_act) || !aligned16(k_cache) ||
        !aligned16(v_cache))
        return JANO_EALIGN;
    int* err = device_error_word();
    if (!err) return JANO_ECUDA;
    const ProjSeg segs[3] = {{q_act, nullptr, hd, n_act}, {k_cache, idx, hd, n_tokens},
                             {v_cache, idx, hd, n_tokens}};
    return from_cuda(launch_projection(x, n_tokens, idx, n_act, w_qkv, 3 * hd, k, 3, segs, err,
                                       static_cast<cudaStream_t>(stream)));
}

jano_status jano_random_scores(int n_blocks, uint64_t seed, float* scores, void* stream) {
    if (n_blocks < 1 || !scores) return JANO_EINVAL;
    return from_cuda(launch_random_scores(n_blocks, seed, scores, static_cast<cudaStream_t>(stream)));
}

jano_status jano_fft_scores(const float* x, int C, const jano_geom* g, int cutoff, float* scores,
                            void* stream) {
    if (!x || !scores || C < 1 || cutoff < 0) return JANO_EINVAL;
    const jano_status gs = check_geom(g, false);
    if (gs != JANO_OK) return gs;
    if ((long long)C * g->F * g->H * g->W > (1ll << 40)) return JANO_EUNSUPPORTED;
    if (!fft_scores_supported(*g)) return JANO_EUNSUPPORTED;
    return from_cuda(launch_fft_scores(x, C, *g, cutoff, scores, static_cast<cudaStream_t>(stream)));
}

jano_status jano_stream_sum(const float* x, long long n, float* partial, int n_partial, void* stream) {
    if (n < 0 || n % 4 || n_partial < 1 || n_partial > 65535 || !partial) return JANO_EINVAL;
    if (n > 0 && !x) return JANO_EINVAL;
    if (!aligned16(x) || !aligned16(partial)) return JANO_EALIGN;
    int* err = device_error_word();
    if (!err) return JANO_ECUDA;
    return from_cuda(launch_stream_sum(x, n, partial, n_partial, err, static_cast<cudaStream_t>(stream)));
}

jano_status jano_get_device_error(void* stream) {
    int* err = device_error_word();
    if (!err) return JANO_ECUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return JANO_ECUDA;
    int v = JANO_OK;
    if (cudaMemcpy(&v, err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return JANO_ECUDA;
    if (v != JANO_OK) {
        const int zero = JANO_OK;
        if (cudaMemcpy(err, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
            return JANO_ECUDA;
    }
    return static_cast<jano_status>(v);
}

const char* jano_status_str(jano_status s) {
    switch (s) {
        case JANO_OK: return "ok";
        case JANO_EINVAL: return "invalid argument";
        case JANO_ESHAPE: return "inconsistent shape";
        case JANO_EALIGN: return "pointer not 16-byte aligned";
        case JANO_EUNSUPPORTED: return "unsupported configuration";
        case JANO_ENONFINITE: return "non-finite score";
        case JANO_EINDEX: return "index or level out of range, or indices not strictly ascending";
        case JANO_ETIMEOUT: return "device wait timed out";
        case JANO_ECUDA: return "CUDA error";
    }
    return "unknown status";
}

int jano_version(void) { return 100; }

}  // extern "C"
