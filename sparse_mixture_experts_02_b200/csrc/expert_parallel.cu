// Expert parallelism: the row movement around ParallelLinear when the experts are spread over
// ranks (ScatterMoE guide, "Combine with Tensor and Pipeline Parallelism": expert weights
// distributed over expert-parallel groups, ScatterMoE handling the local experts). The exchange
// itself is the caller's (NCCL all-to-all over NVLink); these kernels prepare and consume it.
//   pack:      send[p] = x[sorted_rows[p] / k], send_e[p] = top_experts[sorted_rows[p]] for the
//              slots of the sparse map, i.e. the routed rows grouped by expert. Experts of one
//              rank are contiguous, so the rows are grouped by destination rank as well.
//   local ids: the received rows' expert ids relative to this rank's first expert.
//   combine:   out[s] = sum_j w_{s,j} * ret[sparse_rows[s k + j]], the returned expert outputs
//              gathered back per token (no atomics: every token sums its k rows in order).
// One warp per row; rows move in 16-byte pieces.
#include "moe_internal.cuh"

#include <algorithm>

namespace moe {
namespace {

constexpr int kWarps = 8;

int warp_grid(int64_t rows) {
    const int64_t b = (rows + kWarps - 1) / kWarps;
    return (int)std::min<int64_t>(std::max<int64_t>(b, 1), 148LL * 16);
}

__global__ void __launch_bounds__(kWarps * 32)
ep_pack_kernel(const uint4 *__restrict__ x, const int32_t *__restrict__ top_e,
               const int32_t *__restrict__ sorted_rows, const int32_t *__restrict__ offsets,
               int32_t E, int32_t k, int64_t R, int64_t u16, uint4 *__restrict__ send,
               int32_t *__restrict__ send_e, unsigned *status) {
    const int lane = threadIdx.x & 31;
    const int64_t valid = min(R, (int64_t)__ldg(offsets + E));
    const int64_t wstride = (int64_t)gridDim.x * kWarps;
    for (int64_t p = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5); p < valid; p += wstride) {
        const int64_t i = __ldg(sorted_rows + p);
        if (!dev::debug_in_range(i, R, lane == 0 ? status : nullptr)) continue;
        const int64_t s = i / k;
        for (int64_t c = lane; c < u16; c += 32) send[p * u16 + c] = __ldg(x + s * u16 + c);
        if (lane == 0) send_e[p] = __ldg(top_e + i);
    }
}

__global__ void local_ids_kernel(const int32_t *__restrict__ ids, int32_t base, int64_t R,
                                 int32_t *__restrict__ local, unsigned *status) {
    // the first kernel of the receiving side: it clears the status word
    if (blockIdx.x == 0 && threadIdx.x == 0 && status != nullptr) *status = 0u;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < R;
         i += (int64_t)gridDim.x * blockDim.x)
        local[i] = __ldg(ids + i) - base;  // out of range stays out of range: the map flags it
}

__global__ void __launch_bounds__(kWarps * 32)
ep_combine_kernel(const float4 *__restrict__ ret, const int32_t *__restrict__ sparse_rows,
                  const float *__restrict__ w, int64_t S, int32_t k, int64_t R, int64_t d4,
                  float4 *__restrict__ out) {
    const int lane = threadIdx.x & 31;
    const int64_t wstride = (int64_t)gridDim.x * kWarps;
    for (int64_t s = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5); s < S; s += wstride) {
        for (int64_t c = lane; c < d4; c += 32) {
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int j = 0; j < k; ++j) {
                const int64_t p = __ldg(sparse_rows + s * k + j);
                if (p < 0 || p >= R) continue;  // a route whose expert id was out of range
                const float g = __ldg(w + s * k + j);
                const float4 v = __ldg(ret + p * d4 + c);
                acc.x = fmaf(g, v.x, acc.x);
                acc.y = fmaf(g, v.y, acc.y);
                acc.z = fmaf(g, v.z, acc.z);
                acc.w = fmaf(g, v.w, acc.w);
            }
            out[s * d4 + c] = acc;
        }
    }
}

}  // namespace

void launch_ep_pack(const void *x, size_t row_bytes, const int32_t *top_e,
                    const int32_t *sorted_rows, const int32_t *offsets, int32_t E, int32_t k,
                    int64_t R, void *send, int32_t *send_e, unsigned *status, cudaStream_t s) {
    ep_pack_kernel<<<warp_grid(R), kWarps * 32, 0, s>>>(
        static_cast<const uint4 *>(x), top_e, sorted_rows, offsets, E, k, R,
        (int64_t)(row_bytes / 16), static_cast<uint4 *>(send), send_e, status);
}

void launch_local_ids(const int32_t *ids, int32_t base, int64_t R, int32_t *local,
                      unsigned *status, cudaStream_t s) {
    const int64_t b = std::min<int64_t>(std::max<int64_t>((R + 255) / 256, 1), 148LL * 8);
    local_ids_kernel<<<(unsigned)b, 256, 0, s>>>(ids, base, R, local, status);
}

void launch_ep_combine(const float *ret, const int32_t *sparse_rows, const float *w, int64_t S,
                       int32_t k, int64_t R, int64_t D, float *out, cudaStream_t s) {
    ep_combine_kernel<<<warp_grid(S), kWarps * 32, 0, s>>>(
        reinterpret_cast<const float4 *>(ret), sparse_rows, w, S, k, R, D / 4,
        reinterpret_cast<float4 *>(out));
}

}  // namespace moe
