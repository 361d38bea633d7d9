// random_levels.cu -- scores of the random-masking ablation (Jano pages: ko
// technical summary, section 4 "Ablation Study": random masking at a similar
// speed-up, against which the convergence-aware levels give clearly better
// quality).  The ablation keeps the level counts and assigns the levels at
// random; classifying these scores with jano_classify does exactly that.
//
//   scores[b] = (splitmix64 output number b+1 of the stream seeded with seed) >> 40, times 2^-24
//
// splitmix64 (Steele, Lea and Flood, 2014) is counter-based: output i is the
// 64-bit finaliser applied to seed + i * 0x9E3779B97F4A7C15, so every thread
// computes its own block's value with no shared state.  Writes n floats:
// HBM-bound and tiny (77 KB for the large video latent).
#include "jano_common.cuh"

namespace jano {
namespace {

__device__ __forceinline__ uint64_t finalise(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

__global__ void random_scores_kernel(int n, uint64_t seed, float* __restrict__ scores) {
    for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < n; b += gridDim.x * blockDim.x) {
        const uint64_t r = finalise(seed + (uint64_t)(b + 1) * 0x9E3779B97F4A7C15ull);
        scores[b] = (float)(uint32_t)(r >> 40) * 0x1p-24f;     // exact: a 24-bit integer
    }
}

}  // namespace

cudaError_t launch_random_scores(int n, uint64_t seed, float* scores, cudaStream_t st) {
    const int threads = 256;
    int blocks = (n + threads - 1) / threads;
    if (blocks > 4 * 148) blocks = 4 * 148;
    random_scores_kernel<<<blocks, threads, 0, st>>>(n, seed, scores);
    return cudaGetLastError();
}

}  // namespace jano
