// schedule_noalloc.cu -- jano_build_schedule_noalloc: the schedule builder
// for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocating routine) at the
// point where they build the schedule: plug-ins handed fixed buffers by a
// host framework, allocator-less embedded runtimes, or hosts whose memory pool is owned by another framework that forbids side
// allocations.  They still own the inputs and outputs; what they cannot
// provide is the builder's scratch.  This entry point takes its scratch from
// a fixed array in the library's own device image instead, so it allocates
// nothing.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds kStaticScratchBytes of it until the process exits.  In host
// code its name is only a host-side stand-in, not a device address, so the
// real address is fetched with cudaGetSymbolAddress once per device (with
// that device current) the first time the entry point runs there, and that
// address is what the kernels receive.
#include <mutex>

#include "jano_common.cuh"

namespace jano {
namespace {

// 1 MiB: token levels (1 byte per token) plus an int32 [3][tiles] table of
// 1024-token tiles, each part rounded up to 16 bytes; that holds geometries
// of at most 1,036,416 tokens (1,048,576 bytes exactly).
constexpr size_t kStaticScratchBytes = size_t(1) << 20;

static __device__ __align__(256) unsigned char g_schedule_scratch[kStaticScratchBytes];

void* scratch_address(int dev) {
    static std::mutex mu;
    static void* addr[64] = {nullptr};
    if (dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_schedule_scratch) != cudaSuccess) return nullptr;
        addr[dev] = p;
    }
    return addr[dev];
}

}  // namespace
}  // namespace jano

extern "C" JANO_API jano_status jano_build_schedule_noalloc(
    const uint8_t* block_levels, const jano_geom* g, const jano_sched_cfg* c, int32_t* offsets,
    int32_t* idx, size_t idx_capacity, uint8_t* token_levels, void* stream) {
    const size_t need = jano_build_schedule_workspace_bytes(g);   // 0 for an invalid geometry
    if (need > jano::kStaticScratchBytes) return JANO_EUNSUPPORTED;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return JANO_ECUDA;
    void* ws = jano::scratch_address(dev);
    if (!ws) return JANO_ECUDA;
    // Same validation and launches as jano_build_schedule, with the static
    // array as its workspace (the builder needs no zeroed scratch).
    return jano_build_schedule(block_levels, g, c, offsets, idx, idx_capacity, token_levels, ws,
                               jano::kStaticScratchBytes, stream);
}
