// Router: logits = x . W_gate (+ bias), top-k in descending order (ties: smaller expert id),
// softmax over the k selected logits.
//
// ScatterMoE guide ("ScatterMoE Guide: Fast Fused Kernels for Sparse MoE LLMs"),
// "1. The Dynamic Routing Imbalance Dilemma": H(X) = Softmax(TopK(X W_gate, k)).
//
// Layout: one warp owns kTokPerWarp tokens; lane l owns experts e = l + 32 j (j < NJ), so the
// W_gate row loads are coalesced and the logits of a token end up spread over the warp, where the
// top-k is a k-round warp arg-max. x rows are staged through shared memory (fp32) in chunks of 64
// columns, read back as float4 broadcasts. Accumulation is fp32 FMA in ascending d.
#include "moe_internal.cuh"

#include <math.h>

#include <algorithm>
#include <mutex>

namespace moe {
namespace {

constexpr int kTokPerWarp = 8;
constexpr int kWarps = 8;
constexpr int kChunk = 64;
constexpr int kRouteE8MaxSmem = 96 * 1024;  // W_gate rows of the eight-expert router: D <= 6144
constexpr int kE8Batch = 16;                // x pieces a lane has in flight in that router
constexpr int kE8Tokens = 4;                // tokens per warp task of that router

template <bool BF16>
__device__ __forceinline__ float ld_elem(const void *p, int64_t i) {
    if constexpr (BF16) {
        return __bfloat162float(__ldg(reinterpret_cast<const __nv_bfloat16 *>(p) + i));
    } else {
        return __ldg(reinterpret_cast<const float *>(p) + i);
    }
}

// (value, index) is better than (v2, i2): larger value, or equal value and smaller index.
__device__ __forceinline__ bool better(float v, int i, float v2, int i2) {
    return (v > v2) || (v == v2 && i < i2);
}

template <int NJ, bool BF16>
__global__ void __launch_bounds__(kWarps * 32)
route_kernel(const void *__restrict__ x, const void *__restrict__ w_gate,
             const float *__restrict__ bias, int64_t S, int64_t D, int32_t E, int32_t k,
             int32_t *__restrict__ top_e, float *__restrict__ top_w, unsigned *status) {
    __shared__ __align__(16) float xs[kWarps][kTokPerWarp][kChunk];
    if (status != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *status = 0u;  // first kernel
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t tok0 = ((int64_t)blockIdx.x * kWarps + warp) * kTokPerWarp;
    if (tok0 >= S) return;

    float acc[kTokPerWarp][NJ];
#pragma unroll
    for (int t = 0; t < kTokPerWarp; ++t)
#pragma unroll
        for (int j = 0; j < NJ; ++j) acc[t][j] = 0.f;

    for (int64_t d0 = 0; d0 < D; d0 += kChunk) {
        // stage x[tok0 + t][d0 : d0 + 64] as fp32; lane l holds columns 2l, 2l+1
#pragma unroll
        for (int t = 0; t < kTokPerWarp; ++t) {
            const int64_t s = tok0 + t;
            const int64_t c = d0 + 2 * lane;
            float a = 0.f, b = 0.f;
            if (s < S) {
                if (c < D) a = ld_elem<BF16>(x, s * D + c);
                if (c + 1 < D) b = ld_elem<BF16>(x, s * D + c + 1);
            }
            xs[warp][t][2 * lane] = a;
            xs[warp][t][2 * lane + 1] = b;
        }
        __syncwarp();
        const int nd = (D - d0 < kChunk) ? (int)(D - d0) : kChunk;
        for (int d = 0; d < nd; d += 4) {
            float4 xv[kTokPerWarp];
#pragma unroll
            for (int t = 0; t < kTokPerWarp; ++t)
                xv[t] = *reinterpret_cast<const float4 *>(&xs[warp][t][d]);
#pragma unroll
            for (int dd = 0; dd < 4; ++dd) {
                if (d + dd >= nd) break;
                const int64_t row = (d0 + d + dd) * (int64_t)E;
                float w[NJ];
#pragma unroll
                for (int j = 0; j < NJ; ++j) {
                    const int e = lane + 32 * j;
                    w[j] = (e < E) ? ld_elem<BF16>(w_gate, row + e) : 0.f;
                }
#pragma unroll
                for (int t = 0; t < kTokPerWarp; ++t) {
                    const float xd = dd == 0 ? xv[t].x : dd == 1 ? xv[t].y : dd == 2 ? xv[t].z
                                                                                   : xv[t].w;
#pragma unroll
                    for (int j = 0; j < NJ; ++j) acc[t][j] = fmaf(xd, w[j], acc[t][j]);
                }
            }
        }
        __syncwarp();
    }

    // top-k per token: k rounds of a warp arg-max over the lanes' untaken experts
#pragma unroll
    for (int t = 0; t < kTokPerWarp; ++t) {
        const int64_t s = tok0 + t;
        if (s >= S) break;
        float v[NJ];
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
            const int e = lane + 32 * j;
            float l = acc[t][j];
            if (e < E && bias != nullptr) l += __ldg(bias + e);
            if (e >= E || isnan(l)) l = -INFINITY;
            v[j] = l;
        }
        unsigned taken = 0;
        float sel_v[8];
        int sel_i[8];
        for (int r = 0; r < k; ++r) {
            float bv = -INFINITY;
            int bi = 0x7fffffff;
#pragma unroll
            for (int j = 0; j < NJ; ++j) {
                const int e = lane + 32 * j;
                if (e < E && !(taken & (1u << j)) && better(v[j], e, bv, bi)) {
                    bv = v[j];
                    bi = e;
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
                const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
                if (better(ov, oi, bv, bi)) {
                    bv = ov;
                    bi = oi;
                }
            }
            if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
            sel_v[r] = bv;
            sel_i[r] = bi;
        }
        if (lane == 0) {
            const float m = sel_v[0];
            float den = 0.f;
            for (int r = 0; r < k; ++r) den += expf(sel_v[r] - m);
            for (int r = 0; r < k; ++r) {
                top_e[s * k + r] = sel_i[r];
                top_w[s * k + r] = expf(sel_v[r] - m) / den;
            }
        }
    }
}

// Router for E = 8 experts (bf16) at large batches. Persistent blocks stage W_gate [D, 8] (bf16
// rows of 16 bytes) in shared memory once; a warp owns T consecutive tokens at a time, lane l
// reads the 16-byte pieces c = l + 32 j of their x rows (8 consecutive d each, coalesced across
// the warp; kE8Batch pieces in flight over the T rows) and accumulates the T x 8 dot products in
// fp32, ascending d within the lane. Each W_gate row is read from shared memory and widened to
// fp32 once per piece and used for all T tokens. Row d sits at slot d ^ ((d >> 3) & 7): the rows
// of a piece keep their 128 bytes, permuted so that, for a given row offset, the eight lanes of a
// quarter-warp read eight different 16-byte bank groups. The lanes' sums are added by a
// butterfly, after which lane t takes the top-k and the softmax of token t.
template <int T>
__global__ void __launch_bounds__(kWarps * 32)
route_e8_kernel(const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ w_gate,
                const float *__restrict__ bias, int64_t S, int64_t D, int32_t k,
                int32_t *__restrict__ top_e, float *__restrict__ top_w, unsigned *status) {
    constexpr int NE = 8;
    constexpr int B = kE8Batch / T;  // pieces in flight per token row
    static_assert(B * T == kE8Batch && T <= 32, "token group");
    extern __shared__ __align__(16) uint4 wrow[];  // D rows of 8 bf16
    if (status != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *status = 0u;  // first kernel
    const uint4 *wg = reinterpret_cast<const uint4 *>(w_gate);
    for (int64_t d0 = threadIdx.x; d0 < D; d0 += 8 * (int64_t)blockDim.x) {
        uint4 r[8];
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            const int64_t d = d0 + (int64_t)b * blockDim.x;
            if (d < D) r[b] = __ldg(wg + d);
        }
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            const int64_t d = d0 + (int64_t)b * blockDim.x;
            if (d < D) wrow[d ^ ((d >> 3) & 7)] = r[b];
        }
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t pieces = D / 8;
    const int64_t groups = (S + T - 1) / T;
    for (int64_t g = (int64_t)blockIdx.x * kWarps + warp; g < groups;
         g += (int64_t)gridDim.x * kWarps) {
        const int64_t s0 = g * T;
        // experts (2j, 2j+1) of token t accumulate as one float2: a packed two-wide FMA rounds
        // each half exactly like fmaf, so the sums are the same as with scalar FMAs
        float2 acc2[T][NE / 2];
#pragma unroll
        for (int t = 0; t < T; ++t)
#pragma unroll
            for (int j = 0; j < NE / 2; ++j) acc2[t][j] = make_float2(0.f, 0.f);
        // B pieces of each of the T rows are loaded before any is used, so their latencies
        // overlap; a token past S reads zeros
        for (int64_t c0 = lane; c0 < pieces; c0 += 32 * B) {
            uint4 xv[T][B];
#pragma unroll
            for (int t = 0; t < T; ++t) {
                const uint4 *xr = reinterpret_cast<const uint4 *>(x + (s0 + t) * D);
#pragma unroll
                for (int b = 0; b < B; ++b) {
                    const int64_t c = c0 + 32 * b;
                    xv[t][b] = (c < pieces && s0 + t < S) ? __ldg(xr + c)
                                                          : make_uint4(0u, 0u, 0u, 0u);
                }
            }
#pragma unroll
            for (int b = 0; b < B; ++b) {
                const int64_t c = c0 + 32 * b;
                if (c >= pieces) break;
                const int64_t base = 8 * c;
                const int sw = (int)(c & 7);
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    float2 xf[T];
#pragma unroll
                    for (int t = 0; t < T; ++t)
                        xf[t] = __bfloat1622float2(
                            reinterpret_cast<const __nv_bfloat162 *>(&xv[t][b])[h]);
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const int u = 2 * h + q;
                        const uint4 wv = wrow[base + (u ^ sw)];
                        const __nv_bfloat162 *wp = reinterpret_cast<const __nv_bfloat162 *>(&wv);
                        float2 w2[NE / 2];
#pragma unroll
                        for (int j = 0; j < NE / 2; ++j) w2[j] = __bfloat1622float2(wp[j]);
#pragma unroll
                        for (int t = 0; t < T; ++t) {
                            const float xu = q == 0 ? xf[t].x : xf[t].y;
                            const float2 xx = make_float2(xu, xu);
#pragma unroll
                            for (int j = 0; j < NE / 2; ++j)
                                acc2[t][j] = __ffma2_rn(xx, w2[j], acc2[t][j]);
                        }
                    }
                }
            }
        }
        float acc[T][NE];
#pragma unroll
        for (int t = 0; t < T; ++t)
#pragma unroll
            for (int j = 0; j < NE / 2; ++j) {
                acc[t][2 * j] = acc2[t][j].x;
                acc[t][2 * j + 1] = acc2[t][j].y;
            }
#pragma unroll
        for (int t = 0; t < T; ++t)
#pragma unroll
            for (int e = 0; e < NE; ++e)
#pragma unroll
                for (int off = 16; off > 0; off >>= 1)
                    acc[t][e] += __shfl_xor_sync(0xffffffffu, acc[t][e], off);
        // lane t < T finishes token s0 + t (every lane holds every sum after the butterfly)
        float v[NE];
#pragma unroll
        for (int e = 0; e < NE; ++e) {
            float l = acc[0][e];
#pragma unroll
            for (int t = 1; t < T; ++t)
                if (lane == t) l = acc[t][e];
            if (bias != nullptr) l += __ldg(bias + e);
            v[e] = isnan(l) ? -INFINITY : l;
        }
        const int64_t s = s0 + lane;
        if (lane < T && s < S) {
            unsigned taken = 0;
            float sel_v[8];
            int sel_i[8];
            for (int r = 0; r < k; ++r) {
                float bv = -INFINITY;
                int bi = 0x7fffffff;
#pragma unroll
                for (int e = 0; e < NE; ++e)
                    if (!(taken & (1u << e)) && better(v[e], e, bv, bi)) {
                        bv = v[e];
                        bi = e;
                    }
                taken |= 1u << bi;
                sel_v[r] = bv;
                sel_i[r] = bi;
            }
            const float m = sel_v[0];
            float den = 0.f;
            for (int r = 0; r < k; ++r) den += expf(sel_v[r] - m);
            for (int r = 0; r < k; ++r) {
                top_e[s * k + r] = sel_i[r];
                top_w[s * k + r] = expf(sel_v[r] - m) / den;
            }
        }
    }
}

// Router for small batches and few experts (E <= 64): one block per token, so even a decode
// batch spreads over every SM. Thread t accumulates, in fp32 and ascending d within its slice,
// the E partial dot products of d in {8t .. 8t+7} + 1024 j; the block then sums the partials
// (fixed order: warp butterfly, then the four warps in order) and one warp takes the top-k.
template <int NE, bool BF16>
__global__ void __launch_bounds__(128)
route_small_kernel(const void *__restrict__ x, const void *__restrict__ w_gate,
                   const float *__restrict__ bias, int64_t D, int32_t E, int32_t k,
                   int32_t *__restrict__ top_e, float *__restrict__ top_w, unsigned *status) {
    __shared__ float part[4][NE];
    if (status != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *status = 0u;  // first kernel
    const int64_t s = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    float acc[NE];
#pragma unroll
    for (int e = 0; e < NE; ++e) acc[e] = 0.f;
    for (int64_t d0 = (int64_t)tid * 8; d0 < D; d0 += 1024) {
        float xv[8];
        if constexpr (BF16) {
            // 8 consecutive bf16 of x in one 16-byte load (D % 8 == 0, rows 16-byte aligned)
            const uint4 q = __ldg(reinterpret_cast<const uint4 *>(
                reinterpret_cast<const __nv_bfloat16 *>(x) + s * D + d0));
            const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&q);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 f = __bfloat1622float2(h2[j]);
                xv[2 * j] = f.x;
                xv[2 * j + 1] = f.y;
            }
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) xv[j] = ld_elem<BF16>(x, s * D + d0 + j);
        }
        if (BF16 && NE == E) {  // E in {8, 16, 32, 64}: whole 16-byte row pieces
            // rows d0 .. d0+7 of W_gate are 8*E contiguous bf16: E 16-byte loads
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint4 *wr = reinterpret_cast<const uint4 *>(
                    reinterpret_cast<const __nv_bfloat16 *>(w_gate) + (d0 + j) * (int64_t)E);
#pragma unroll
                for (int c = 0; c < NE / 8; ++c) {
                    const uint4 q = __ldg(wr + c);
                    const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&q);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float2 f = __bfloat1622float2(h2[u]);
                        acc[c * 8 + 2 * u] = fmaf(xv[j], f.x, acc[c * 8 + 2 * u]);
                        acc[c * 8 + 2 * u + 1] = fmaf(xv[j], f.y, acc[c * 8 + 2 * u + 1]);
                    }
                }
            }
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int64_t row = (d0 + j) * (int64_t)E;
#pragma unroll
                for (int e = 0; e < NE; ++e)
                    if (e < E) acc[e] = fmaf(xv[j], ld_elem<BF16>(w_gate, row + e), acc[e]);
            }
        }
    }
#pragma unroll
    for (int e = 0; e < NE; ++e) {
        float v = acc[e];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == 0) part[warp][e] = v;
    }
    __syncthreads();
    if (warp != 0) return;
    // lane l owns experts l and l + 32
    float v[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int e = lane + 32 * h;
        float l = -INFINITY;
        if (e < E && e < NE) {
            l = ((part[0][e] + part[1][e]) + part[2][e]) + part[3][e];
            if (bias != nullptr) l += __ldg(bias + e);
            if (isnan(l)) l = -INFINITY;
        }
        v[h] = l;
    }
    unsigned taken = 0;
    float sel_v[8];
    int sel_i[8];
    for (int r = 0; r < k; ++r) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int e = lane + 32 * h;
            if (e < E && !(taken & (1u << h)) && better(v[h], e, bv, bi)) {
                bv = v[h];
                bi = e;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
            if (better(ov, oi, bv, bi)) {
                bv = ov;
                bi = oi;
            }
        }
        if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
        sel_v[r] = bv;
        sel_i[r] = bi;
    }
    if (lane == 0) {
        const float m = sel_v[0];
        float den = 0.f;
        for (int r = 0; r < k; ++r) den += expf(sel_v[r] - m);
        for (int r = 0; r < k; ++r) {
            top_e[s * k + r] = sel_i[r];
            top_w[s * k + r] = expf(sel_v[r] - m) / den;
        }
    }
}

template <int NE>
void launch_route_small_ne(const void *x, const void *w_gate, const float *bias, int64_t S,
                           int64_t D, int32_t E, int32_t k, bool bf16, int32_t *top_e,
                           float *top_w, unsigned *status, cudaStream_t s) {
    if (bf16)
        route_small_kernel<NE, true><<<(unsigned)S, 128, 0, s>>>(x, w_gate, bias, D, E, k, top_e,
                                                                 top_w, status);
    else
        route_small_kernel<NE, false><<<(unsigned)S, 128, 0, s>>>(x, w_gate, bias, D, E, k,
                                                                  top_e, top_w, status);
}

__global__ void zero_kernel(float4 *__restrict__ p, int64_t n4, float *__restrict__ tail,
                            int tail_n, unsigned *status) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride)
        p[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (blockIdx.x == 0 && threadIdx.x < tail_n) tail[threadIdx.x] = 0.f;
    if (blockIdx.x == 0 && threadIdx.x == 0 && status != nullptr) *status = 0u;
}

template <int NJ>
int launch_route_nj(const void *x, const void *w_gate, const float *bias, int64_t S, int64_t D,
                    int32_t E, int32_t k, bool bf16, int32_t *top_e, float *top_w,
                    unsigned *status, cudaStream_t s) {
    const int64_t per_block = (int64_t)kWarps * kTokPerWarp;
    const int64_t blocks = (S + per_block - 1) / per_block;
    if (blocks == 0) return 0;
    if (bf16)
        route_kernel<NJ, true><<<(unsigned)blocks, kWarps * 32, 0, s>>>(x, w_gate, bias, S, D, E,
                                                                        k, top_e, top_w, status);
    else
        route_kernel<NJ, false><<<(unsigned)blocks, kWarps * 32, 0, s>>>(x, w_gate, bias, S, D,
                                                                         E, k, top_e, top_w,
                                                                         status);
    return 1;
}

}  // namespace

int launch_route(const void *x, const void *w_gate, const float *bias, int64_t S, int64_t D,
                 int32_t E, int32_t k, bool bf16, int32_t *top_e, float *top_w, unsigned *status,
                 cudaStream_t s) {
    if (S == 0) return 0;
    // Eight experts (bf16), a batch too large for one block per token: W_gate fits in shared
    // memory and every SM streams x rows (measured 20 us with x in L2, against 29 us for the
    // tensor-core router, at S = 4096, D = 4096).
    if (bf16 && E == 8 && S > 2048 && D * 16 <= kRouteE8MaxSmem) {
        static std::once_flag once;
        static cudaError_t attr_err = cudaSuccess;
        std::call_once(once, [] {
            attr_err = cudaFuncSetAttribute(route_e8_kernel<kE8Tokens>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            kRouteE8MaxSmem);
        });
        if (attr_err != cudaSuccess) {
            set_error(MOE_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(attr_err));
            return -1;
        }
        const int64_t want = (S + kE8Tokens * kWarps - 1) / (kE8Tokens * kWarps);
        const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>(want, 2LL * num_sms()));
        route_e8_kernel<kE8Tokens><<<(unsigned)blocks, kWarps * 32, (size_t)(D * 16), s>>>(
            static_cast<const __nv_bfloat16 *>(x), static_cast<const __nv_bfloat16 *>(w_gate),
            bias, S, D, k, top_e, top_w, status);
        return 1;
    }
    // Few experts and a batch too small to fill the SMs with 128-token tensor-core tiles (or fp32
    // inputs): one block per token on the CUDA cores, exact fp32 accumulation.
    if (E <= 64 && (S <= 2048 || !bf16) && S < (int64_t(1) << 31)) {
        if (E <= 8) launch_route_small_ne<8>(x, w_gate, bias, S, D, E, k, bf16, top_e, top_w, status, s);
        else if (E <= 16) launch_route_small_ne<16>(x, w_gate, bias, S, D, E, k, bf16, top_e, top_w, status, s);
        else if (E <= 32) launch_route_small_ne<32>(x, w_gate, bias, S, D, E, k, bf16, top_e, top_w, status, s);
        else launch_route_small_ne<64>(x, w_gate, bias, S, D, E, k, bf16, top_e, top_w, status, s);
        return 1;
    }
    // bf16 with E a multiple of 8 (16-byte W_gate rows for TMA): tensor-core router.
    // Otherwise (fp32 inputs, or odd E): exact fp32 FMA accumulation on the CUDA cores.
    if (bf16 && E % 8 == 0) {
        if (launch_route_tc(x, w_gate, bias, S, D, E, k, top_e, top_w, status, s) != MOE_OK)
            return -1;
        return 1;
    }
    if (E <= 32) return launch_route_nj<1>(x, w_gate, bias, S, D, E, k, bf16, top_e, top_w, status, s);
    if (E <= 64) return launch_route_nj<2>(x, w_gate, bias, S, D, E, k, bf16, top_e, top_w, status, s);
    if (E <= 128) return launch_route_nj<4>(x, w_gate, bias, S, D, E, k, bf16, top_e, top_w, status, s);
    return launch_route_nj<8>(x, w_gate, bias, S, D, E, k, bf16, top_e, top_w, status, s);
}

int launch_zero_f32(float *p, int64_t n, unsigned *status, cudaStream_t s) {
    // p is 16-byte aligned (checked by the caller); n4 float4 stores plus a < 4 element tail
    const int64_t n4 = n / 4;
    const int tail = (int)(n - n4 * 4);
    int64_t blocks = (n4 + 255) / 256;
    const int64_t cap = (int64_t)num_sms() * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    zero_kernel<<<(unsigned)blocks, 256, 0, s>>>(reinterpret_cast<float4 *>(p), n4, p + n4 * 4,
                                                  tail, status);
    return 1;
}

}  // namespace moe
