// Elementwise and row-reduction kernels of the ParallelLinear backward (ScatterMoE guide,
// "3. Fused Backward Pass Dynamics"); the GEMMs are the tensor-core kernels of grouped_gemm.cu
// (input gradient: the forward's form with W read transposed) and grouped_gemm_wgrad.cu (weight
// gradient).
//   cast:      an fp32 output gradient [rows, Dout] -> bf16 (the tensor cores' operand type);
//   gate_rows: dv[p] = bf16(g_i * dY[row(p)]), the weight gradient's B operand, in slot order or
//              in its padded layout (row p + 64 e(p); row(p) = sorted_rows[p] / k when the forward
//              scattered into tokens, else p); zero_pad_rows zeroes that layout's padding rows;
//   gather_rows: x rows in slot order (the weight gradient's A operand for gathered inputs);
//   rowdot:    dgates[i] = sum_n dY[row(p)][n] * v[p][n], v = the ungated forward rows.
// One warp per slot; rows move in 16-byte pieces (Dout is a multiple of 8).
#include "moe_internal.cuh"

#include <cuda_bf16.h>

namespace moe {
namespace {

constexpr int kWarps = 8;

__device__ __forceinline__ void load8(const void *row, bool bf16, int64_t c, float (&v)[8]) {
    if (bf16) {
        const uint4 u = *reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(row) + c);
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 f = __bfloat1622float2(h[j]);
            v[2 * j] = f.x;
            v[2 * j + 1] = f.y;
        }
    } else {
        const float4 a = *reinterpret_cast<const float4 *>(static_cast<const float *>(row) + c);
        const float4 b = *reinterpret_cast<const float4 *>(static_cast<const float *>(row) + c + 4);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
}

__device__ __forceinline__ uint4 pack8(const float (&v)[8]) {
    uint4 u;
    uint32_t *w = reinterpret_cast<uint32_t *>(&u);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        __nv_bfloat162 t = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
        w[j] = *reinterpret_cast<uint32_t *>(&t);
    }
    return u;
}

// Expert of slot p: the largest e with offsets[e] <= p (empty experts share their start with the
// next one, which is the one that holds p).
__device__ __forceinline__ int expert_of(const int32_t *__restrict__ offsets, int32_t E, int64_t p) {
    int lo = 0, hi = E;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(offsets + mid) <= p) lo = mid;
        else hi = mid;
    }
    return lo;
}

__global__ void cast_bf16_kernel(const float *__restrict__ src, __nv_bfloat16 *__restrict__ dst,
                                 int64_t n8) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += stride) {
        float v[8];
        load8(src, false, i * 8, v);
        *reinterpret_cast<uint4 *>(dst + i * 8) = pack8(v);
    }
}

__global__ void __launch_bounds__(kWarps * 32)
gate_rows_kernel(const void *__restrict__ dY, bool dy_bf16, const int32_t *__restrict__ sorted_rows,
                 const float *__restrict__ gates, int32_t k, int64_t R, int64_t Dout,
                 bool by_token, __nv_bfloat16 *__restrict__ dv,
                 const int32_t *__restrict__ pad_offsets, int32_t E, unsigned *status) {
    const int lane = threadIdx.x & 31;
    const int64_t wstride = (int64_t)gridDim.x * kWarps;
    for (int64_t p = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5); p < R; p += wstride) {
        const int32_t i = __ldg(sorted_rows + p);
        if (!dev::debug_in_range(i, R, lane == 0 ? status : nullptr)) continue;
        const float g = gates != nullptr ? __ldg(gates + i) : 1.0f;
        const int64_t row = by_token ? (int64_t)(i / k) : p;
        const uint8_t *src = static_cast<const uint8_t *>(dY) + row * Dout * (dy_bf16 ? 2 : 4);
        const int64_t out = pad_offsets != nullptr ? p + (int64_t)kWgradPad * expert_of(pad_offsets, E, p)
                                                   : p;
        for (int64_t c = (int64_t)lane * 8; c < Dout; c += 32 * 8) {
            float v[8];
            load8(src, dy_bf16, c, v);
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] *= g;
            *reinterpret_cast<uint4 *>(dv + out * Dout + c) = pack8(v);
        }
    }
}

__global__ void __launch_bounds__(kWarps * 32)
rowdot_kernel(const void *__restrict__ dY, bool dy_bf16, const __nv_bfloat16 *__restrict__ v,
              const int32_t *__restrict__ sorted_rows, int32_t k, int64_t R, int64_t Dout,
              bool by_token, float *__restrict__ dg, unsigned *status) {
    const int lane = threadIdx.x & 31;
    const int64_t wstride = (int64_t)gridDim.x * kWarps;
    for (int64_t p = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5); p < R; p += wstride) {
        const int32_t i = __ldg(sorted_rows + p);
        if (!dev::debug_in_range(i, R, lane == 0 ? status : nullptr)) continue;
        const int64_t row = by_token ? (int64_t)(i / k) : p;
        const uint8_t *src = static_cast<const uint8_t *>(dY) + row * Dout * (dy_bf16 ? 2 : 4);
        float acc = 0.f;
        for (int64_t c = (int64_t)lane * 8; c < Dout; c += 32 * 8) {
            float a[8], b[8];
            load8(src, dy_bf16, c, a);
            load8(v + p * Dout, true, c, b);
#pragma unroll
            for (int j = 0; j < 8; ++j) acc = fmaf(a[j], b[j], acc);
        }
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, d);
        if (lane == 0) dg[i] = acc;
    }
}

// Router backward of one token s: the softmax over its k selected logits gives
//   dl_j = w_j (dw_j - sum_j' w_j' dw_j');
// dl is written as a dense bf16 row [E] (zero outside the selection, the weight gradient's
// operand) and dx[s] += sum_j dl_j W_gate[:, e_j] (after the expert part of dx is complete),
// read from W_gate^T [E, D] so that the lanes' loads are consecutive.
// The W_gate gradient splits the tokens into P chunks of `chunk` consecutive tokens (partial
// gradients, summed afterwards): dl rows go to the padded layout of those chunks (token s at
// row s + 64 (s / chunk)), and block 0 writes the chunk offsets min(j chunk, S), j = 0..P.
__global__ void __launch_bounds__(kWarps * 32)
router_bwd_kernel(const int32_t *__restrict__ top_e, const float *__restrict__ top_w,
                  const float *__restrict__ dw, const __nv_bfloat16 *__restrict__ w_gate_t,
                  int64_t S, int64_t D, int32_t E, int32_t k, __nv_bfloat16 *__restrict__ dl,
                  float *__restrict__ dx, int32_t *__restrict__ chunk_offsets, int32_t chunk,
                  int32_t P) {
    const int lane = threadIdx.x & 31;
    if (blockIdx.x == 0)
        for (int j = threadIdx.x; j <= P; j += blockDim.x)
            chunk_offsets[j] = (int32_t)((int64_t)j * chunk < S ? (int64_t)j * chunk : S);
    const int64_t wstride = (int64_t)gridDim.x * kWarps;
    for (int64_t s = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5); s < S; s += wstride) {
        float mean = 0.f;
        for (int j = 0; j < k; ++j) mean += top_w[s * k + j] * dw[s * k + j];
        float dlj[8];
        int32_t ej[8];
        for (int j = 0; j < k; ++j) {
            dlj[j] = top_w[s * k + j] * (dw[s * k + j] - mean);
            ej[j] = top_e[s * k + j];
        }
        const int64_t drow = s + (int64_t)kWgradPad * (s / chunk);
        for (int e = lane; e < E; e += 32) {
            float v = 0.f;
            for (int j = 0; j < k; ++j)
                if (ej[j] == e) v = dlj[j];
            dl[drow * E + e] = __float2bfloat16_rn(v);
        }
        for (int64_t d = lane; d < D; d += 32) {
            float acc = 0.f;
            for (int j = 0; j < k; ++j)
                acc = fmaf(dlj[j], __bfloat162float(w_gate_t[(int64_t)ej[j] * D + d]), acc);
            dx[s * D + d] += acc;
        }
    }
}

// Padding rows of expert e (blockIdx.x) in the padded layout: rows offsets[e] + 64 e + n_e up to
// offsets[e] + 64 e + roundup(n_e, 64) are zeroed, by gridDim.y blocks per expert.
__global__ void zero_pad_rows_kernel(uint4 *__restrict__ rows, int64_t ld16, int64_t cols16,
                                     const int32_t *__restrict__ offsets) {
    const int e = blockIdx.x;
    const int64_t n = __ldg(offsets + e + 1) - __ldg(offsets + e);
    const int64_t first = __ldg(offsets + e) + (int64_t)kWgradPad * e + n;
    const int64_t count = (n + kWgradPad - 1) / kWgradPad * kWgradPad - n;
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    for (int64_t q = (int64_t)blockIdx.y * blockDim.x + threadIdx.x; q < count * cols16;
         q += (int64_t)gridDim.y * blockDim.x)
        rows[(first + q / cols16) * ld16 + q % cols16] = z;
}

// xs[p] = x[sorted_rows[p] / k], bf16 rows of D elements, one warp per slot.
__global__ void __launch_bounds__(kWarps * 32)
gather_rows_kernel(const uint4 *__restrict__ x, const int32_t *__restrict__ sorted_rows, int32_t k,
                   int64_t R, int64_t d16, uint4 *__restrict__ xs, unsigned *status) {
    const int lane = threadIdx.x & 31;
    const int64_t wstride = (int64_t)gridDim.x * kWarps;
    for (int64_t p = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5); p < R; p += wstride) {
        const int32_t i = __ldg(sorted_rows + p);
        if (!dev::debug_in_range(i, R, lane == 0 ? status : nullptr)) continue;
        const int64_t s = i / k;
        for (int64_t c = lane; c < d16; c += 32) xs[p * d16 + c] = __ldg(x + s * d16 + c);
    }
}

// dst [cols, rows] = src [rows, cols]^T (bf16), through 32 x 33 shared tiles.
__global__ void transpose_bf16_kernel(const __nv_bfloat16 *__restrict__ src, int64_t rows,
                                      int64_t cols, __nv_bfloat16 *__restrict__ dst) {
    __shared__ __nv_bfloat16 tile[32][33];
    const int64_t r0 = (int64_t)blockIdx.y * 32, c0 = (int64_t)blockIdx.x * 32;
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int64_t r = r0 + i, c = c0 + threadIdx.x;
        if (r < rows && c < cols) tile[i][threadIdx.x] = src[r * cols + c];
    }
    __syncthreads();
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int64_t c = c0 + i, r = r0 + threadIdx.x;
        if (c < cols && r < rows) dst[c * rows + r] = tile[threadIdx.x][i];
    }
}

// out[i] = sum over j < P of partial[j][i], i < n (the chunks' partial W_gate gradients).
__global__ void sum_partials_kernel(const float *__restrict__ partial, int64_t n, int32_t P,
                                    float *__restrict__ out) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        float acc = 0.f;
        for (int j = 0; j < P; ++j) acc += partial[(int64_t)j * n + i];
        out[i] = acc;
    }
}

unsigned warp_grid(int64_t rows) {
    int64_t blocks = (rows + kWarps - 1) / kWarps;
    const int64_t cap = (int64_t)num_sms() * 16;
    if (blocks > cap) blocks = cap;
    return (unsigned)(blocks < 1 ? 1 : blocks);
}

}  // namespace

void launch_cast_bf16(const float *src, void *dst, int64_t n, cudaStream_t s) {
    const int64_t n8 = n / 8;
    int64_t blocks = (n8 + 255) / 256;
    const int64_t cap = (int64_t)num_sms() * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    cast_bf16_kernel<<<(unsigned)blocks, 256, 0, s>>>(src, static_cast<__nv_bfloat16 *>(dst), n8);
}

void launch_gate_rows(const void *dY, bool dy_bf16, const int32_t *sorted_rows, const float *gates,
                      int32_t k, int64_t R, int64_t Dout, bool by_token, void *dv,
                      const int32_t *pad_offsets, int32_t E, unsigned *status, cudaStream_t s) {
    gate_rows_kernel<<<warp_grid(R), kWarps * 32, 0, s>>>(dY, dy_bf16, sorted_rows, gates, k, R,
                                                          Dout, by_token,
                                                          static_cast<__nv_bfloat16 *>(dv),
                                                          pad_offsets, E, status);
}

void launch_zero_pad_rows(void *rows, int64_t ld, int64_t cols, const int32_t *offsets, int32_t E,
                          cudaStream_t s) {
    // up to 63 rows per expert: spread each expert's rows over several blocks
    const int64_t per_expert = 63 * (cols / 8);
    int64_t ys = (per_expert + 4095) / 4096;
    if (ys > 32) ys = 32;
    const dim3 grid((unsigned)E, (unsigned)(ys < 1 ? 1 : ys));
    zero_pad_rows_kernel<<<grid, 256, 0, s>>>(static_cast<uint4 *>(rows), ld / 8, cols / 8,
                                              offsets);
}

void launch_gather_rows(const void *x, const int32_t *sorted_rows, int32_t k, int64_t R, int64_t D,
                        void *xs, unsigned *status, cudaStream_t s) {
    gather_rows_kernel<<<warp_grid(R), kWarps * 32, 0, s>>>(static_cast<const uint4 *>(x),
                                                            sorted_rows, k, R, D / 8,
                                                            static_cast<uint4 *>(xs), status);
}

void launch_rowdot(const void *dY, bool dy_bf16, const void *v, const int32_t *sorted_rows,
                   int32_t k, int64_t R, int64_t Dout, bool by_token, float *dg, unsigned *status,
                   cudaStream_t s) {
    rowdot_kernel<<<warp_grid(R), kWarps * 32, 0, s>>>(dY, dy_bf16,
                                                       static_cast<const __nv_bfloat16 *>(v),
                                                       sorted_rows, k, R, Dout, by_token, dg,
                                                       status);
}

void launch_router_bwd(const int32_t *top_e, const float *top_w, const float *dw,
                       const void *w_gate, void *w_gate_t, int64_t S, int64_t D, int32_t E,
                       int32_t k, void *dl, float *dx, int32_t *chunk_offsets, int32_t chunk,
                       int32_t P, cudaStream_t s) {
    const dim3 grid((unsigned)((E + 31) / 32), (unsigned)((D + 31) / 32));
    transpose_bf16_kernel<<<grid, dim3(32, 8), 0, s>>>(static_cast<const __nv_bfloat16 *>(w_gate),
                                                       D, E,
                                                       static_cast<__nv_bfloat16 *>(w_gate_t));
    router_bwd_kernel<<<warp_grid(S), kWarps * 32, 0, s>>>(
        top_e, top_w, dw, static_cast<const __nv_bfloat16 *>(w_gate_t), S, D, E, k,
        static_cast<__nv_bfloat16 *>(dl), dx, chunk_offsets, chunk, P);
}

void launch_sum_partials(const float *partial, int64_t n, int32_t P, float *out, cudaStream_t s) {
    int64_t blocks = (n + 255) / 256;
    const int64_t cap = (int64_t)num_sms() * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    sum_partials_kernel<<<(unsigned)blocks, 256, 0, s>>>(partial, n, P, out);
}

}  // namespace moe
