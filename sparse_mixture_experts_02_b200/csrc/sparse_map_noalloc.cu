// moe_sparse_map_noalloc: the sparse map for callers that cannot provide device scratch memory.
//
// Some callers can hand the library their input and output buffers but have no way to obtain any
// further device memory at call time: plugin-style interfaces that only pass fixed input/output
// bindings, or runtimes that reserve all device memory in their own pool at start-up, where a
// cudaMalloc for scratch would fail (no free memory left) or stall every stream of the device
// (cudaMalloc may synchronise). For them this entry point keeps its scratch in a fixed-size
// array that is part of the library image itself, so the call allocates nothing.
//
// The array (kNoallocScratchBytes of map scratch plus a 256-byte status area) exists once per
// device that loads the library and stays allocated until the process exits. Its device address
// is looked up once per device, with that device current, on the first call on that device; make
// that first call before any stream capture. With CUDA's lazy module loading (the default), that
// first call may be what loads this module on the device and so reserves the array: make it
// before a memory pool reserves the rest of the device. Every call shares the one array and it keeps the
// last call's contents: the map kernels overwrite every scratch word they later read, and the
// status word is cleared by each call. Two calls whose kernels overlap on the GPU (for example on
// two streams) race on the array and must be serialised by the caller.
#include "moe_internal.cuh"

#include <mutex>

namespace moe {
namespace {

constexpr size_t kNoallocScratchBytes = size_t(1) << 20;  // 1 MiB of per-(unit, expert) counters
constexpr size_t kNoallocBytes = kStatusBytes + kNoallocScratchBytes;

// [0, 256): status word; [256, 256 + 1 MiB): map scratch.
static __device__ __align__(256) unsigned char g_map_scratch[kNoallocBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_addr[kMaxDevices] = {};

// Device address of g_map_scratch on the current device (looked up once per device).
int scratch_address(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return set_error(MOE_ERR_CUDA, "sparse_map_noalloc: no usable current device");
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_addr[dev] == nullptr) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_map_scratch);
        if (e != cudaSuccess || p == nullptr)
            return set_error(MOE_ERR_CUDA, "sparse_map_noalloc: cudaGetSymbolAddress failed: %s",
                             cudaGetErrorString(e));
        g_addr[dev] = p;
    }
    *out = g_addr[dev];
    return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" int moe_sparse_map_noalloc(const int32_t *top_experts, int64_t S, int32_t k, int32_t E,
                                      int32_t *expert_counts, int32_t *expert_offsets,
                                      int32_t *sparse_rows, int32_t *sorted_rows,
                                      moe_stream_t stream) {
    if (S < 0) return set_error(MOE_ERR_INVALID_ARG, "S must be >= 0 (got %lld)", (long long)S);
    if (E < 1 || E > 256) return set_error(MOE_ERR_INVALID_ARG, "E must be in [1, 256] (got %d)", E);
    if (k < 1 || k > 8 || k > E)
        return set_error(MOE_ERR_INVALID_ARG, "k must be in [1, min(E, 8)] (got k=%d, E=%d)", k, E);
    if (S * (int64_t)k >= (int64_t(1) << 31))
        return set_error(MOE_ERR_INVALID_ARG, "S*k must be < 2^31");
    const int64_t R = S * k;
    const size_t need = map_scratch_bytes(R, E);
    if (need > kNoallocScratchBytes)
        return set_error(MOE_ERR_INVALID_ARG,
                         "sparse_map_noalloc: S*k=%lld routes over E=%d experts need %zu bytes of "
                         "scratch, above its fixed %zu bytes ((ceil(S*k/4096)+1)*E*4 must be <= %zu); "
                         "use moe_sparse_map with a workspace",
                         (long long)R, E, need, kNoallocScratchBytes, kNoallocScratchBytes);
    const struct { const char *name; const void *p; bool nullable; } ptrs[] = {
        {"top_experts", top_experts, R == 0}, {"expert_counts", expert_counts, false},
        {"expert_offsets", expert_offsets, false}, {"sparse_rows", sparse_rows, R == 0},
        {"sorted_rows", sorted_rows, R == 0}};
    for (const auto &q : ptrs) {
        if (q.p == nullptr && !q.nullable)
            return set_error(MOE_ERR_INVALID_ARG, "%s is null", q.name);
        if (q.p != nullptr && (reinterpret_cast<uintptr_t>(q.p) & 3u))
            return set_error(MOE_ERR_INVALID_ARG, "%s is not 4-byte aligned", q.name);
    }
    int dev = 0, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return set_error(MOE_ERR_CUDA, "cudaGetDevice failed");
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0)
        return set_error(MOE_ERR_UNSUPPORTED, "this library is built for sm_100a (B200) only");
    void *base = nullptr;
    int rc = scratch_address(&base);
    if (rc) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    unsigned *status = static_cast<unsigned *>(base);
    // the status word accumulates flags with atomicOr: clear it for this call
    if (cudaMemsetAsync(status, 0, sizeof(unsigned), s) != cudaSuccess)
        return set_error(MOE_ERR_CUDA, "sparse_map_noalloc: clearing the status word failed");
    int n = 0;
    launch_sparse_map(top_experts, R, E, expert_counts, expert_offsets, sparse_rows, sorted_rows,
                      reinterpret_cast<int32_t *>(static_cast<unsigned char *>(base) + kStatusBytes),
                      status, s, &n);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return set_error(MOE_ERR_CUDA, "sparse_map_noalloc launch: %s", cudaGetErrorString(e));
    return MOE_OK;
}
