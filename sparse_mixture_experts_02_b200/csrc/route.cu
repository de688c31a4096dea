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
constexpr int kRouteE8MaxSmem = 200 * 1024;  // eight-expert router: padded W_gate, D <= 9792

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

// Router for E = 8 experts (bf16) at large batches, on warp-level tensor-core MMAs
// (mma.sync m16n8k16, bf16 inputs, fp32 accumulation): the router streams x once from HBM, and an
// MMA turns 16 tokens x 16 d x 8 experts of products into one instruction, where fp32 FMAs need
// 64 (the CUDA-core form of this kernel issued ~6 M warp instructions at S = D = 4096 and ran at
// a fifth of HBM bandwidth). A block of 8 warps routes 16 tokens; warp w takes the d range
// [w P / 8, (w + 1) P / 8) of the P = ceil(D / 32) groups of 32 d.
//
// The d order inside one MMA is free (a dot product is a sum), so the fragments come straight
// from coalesced 16-byte loads: lane (g = lane / 4, q = lane % 4) loads d = 32 p + 8 q .. + 7 of
// tokens g and g + 8, and MMA j (0, 1) of group p sums, for that lane's k slots {2q, 2q+1} and
// {2q+8, 2q+9}, the d = 32 p + 8 q + 4 j + {0, 1} and + {2, 3}. The B fragments (W_gate column
// g at the same d) of both MMAs come from one ldmatrix.x4.trans over W_gate rows (16 bytes: the 8
// experts of one d) staged by cp.async in shared memory: each lane names the row of the d its
// k slot stands for, and row d sits at slot d + 2 (d / 8), which puts the 8 rows of every 8 x 8
// matrix on 8 different 16-byte bank groups. Rows past D are zero. The warps' partial logits are
// added in warp order, then one thread per token takes the top-k and the softmax.
constexpr int kE8MmaTokens = 16;
constexpr int kE8MmaUnroll = 8;  // groups of 32 d whose x a lane has in flight

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Shared memory of the eight-expert router: W_gate rows of the ceil(D / 32) groups of 32 d at
// slot d + 2 (d / 8) (40 slots of 16 bytes per group), then the warps' partial logits.
__host__ __device__ constexpr size_t route_e8_smem(int64_t D) {
    return (size_t)((D + 31) / 32) * 40 * 16 + (size_t)kWarps * kE8MmaTokens * 8 * sizeof(float);
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr)
                 : "memory");
}

__global__ void __launch_bounds__(kWarps * 32, 2)
route_e8_kernel(const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ w_gate,
                const float *__restrict__ bias, int64_t S, int64_t D, int32_t k,
                int32_t *__restrict__ top_e, float *__restrict__ top_w, unsigned *status) {
    constexpr int U = kE8MmaUnroll;
    extern __shared__ __align__(16) uint8_t e8_smem[];
    const int Di = (int)D;
    const int P = (Di + 31) / 32;
    float *part = reinterpret_cast<float *>(e8_smem + (size_t)P * 40 * 16);
    if (status != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *status = 0u;  // first kernel
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, q = lane & 3;
    const int64_t t0 = (int64_t)blockIdx.x * kE8MmaTokens;
    const int p0 = warp * P / kWarps, p1 = (warp + 1) * P / kWarps;
    const bool r0 = t0 + g < S, r1 = t0 + g + 8 < S;
    const uint4 *x0 = reinterpret_cast<const uint4 *>(x + (r0 ? t0 + g : 0) * D);
    const uint4 *x1 = reinterpret_cast<const uint4 *>(x + (r1 ? t0 + g + 8 : 0) * D);
    uint4 xa[U], xb[U];
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    auto load = [&](int p) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int c = 4 * (p + u) + q;  // 16-byte piece: d = 8 c .. 8 c + 7
            const bool ok = p + u < p1 && 8 * c < Di;
            xa[u] = ok && r0 ? __ldg(x0 + c) : z;
            xb[u] = ok && r1 ? __ldg(x1 + c) : z;
        }
    };
    // W_gate rows by cp.async (no registers held), then the first x batch: both in flight at once
    const uint32_t wbase = dev::smem_u32(e8_smem);
    const uint4 *wg = reinterpret_cast<const uint4 *>(w_gate);
    for (int d = threadIdx.x; d < 32 * P; d += blockDim.x) {
        const uint32_t dst = wbase + (uint32_t)(d + 2 * (d >> 3)) * 16u;
        dev::cp_async16(dst, d < Di ? wg + d : wg, d < Di ? 16u : 0u);  // rows past D: zeros
    }
    load(p0);
    dev::cp_async_wait_all();
    __syncthreads();
    // ldmatrix row of this lane: matrix m = lane / 8 (MMA j = m / 2, k half m % 2), row r = lane % 8
    const int lm = lane >> 3, lr = lane & 7;
    const int drow = 8 * (lr >> 1) + 4 * (lm >> 1) + 2 * (lm & 1) + (lr & 1);  // d within a group
    float c[4] = {0.f, 0.f, 0.f, 0.f};
    for (int p = p0; p < p1; p += U) {
        if (p != p0) load(p);
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (p + u >= p1) break;
            const int d = 32 * (p + u) + drow;
            uint32_t bw[4];
            ldmatrix_x4_trans(wbase + (uint32_t)(d + 2 * (d >> 3)) * 16u, bw);
            mma_bf16_16816(c, xa[u].x, xb[u].x, xa[u].y, xb[u].y, bw[0], bw[1]);
            mma_bf16_16816(c, xa[u].z, xb[u].z, xa[u].w, xb[u].w, bw[2], bw[3]);
        }
    }
    // c[0], c[1]: token g, experts 2q, 2q+1; c[2], c[3]: token g + 8
    float *pw = part + (size_t)warp * kE8MmaTokens * 8;
    pw[g * 8 + 2 * q] = c[0];
    pw[g * 8 + 2 * q + 1] = c[1];
    pw[(g + 8) * 8 + 2 * q] = c[2];
    pw[(g + 8) * 8 + 2 * q + 1] = c[3];
    __syncthreads();
    if (threadIdx.x < kE8MmaTokens) {
        const int r = threadIdx.x;
        const int64_t s = t0 + r;
        if (s < S) {
            float v[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                float l = part[r * 8 + e];
#pragma unroll
                for (int w = 1; w < kWarps; ++w) l += part[(w * kE8MmaTokens + r) * 8 + e];
                if (bias != nullptr) l += __ldg(bias + e);
                v[e] = isnan(l) ? -INFINITY : l;
            }
            unsigned taken = 0;
            float sel_v[8];
            int sel_i[8];
            for (int rr = 0; rr < k; ++rr) {
                float bv = -INFINITY;
                int bi = 0x7fffffff;
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    if (!(taken & (1u << e)) && better(v[e], e, bv, bi)) {
                        bv = v[e];
                        bi = e;
                    }
                taken |= 1u << bi;
                sel_v[rr] = bv;
                sel_i[rr] = bi;
            }
            const float m = sel_v[0];
            float den = 0.f;
            for (int rr = 0; rr < k; ++rr) den += expf(sel_v[rr] - m);
            for (int rr = 0; rr < k; ++rr) {
                top_e[s * k + rr] = sel_i[rr];
                top_w[s * k + rr] = expf(sel_v[rr] - m) / den;
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
    // Eight experts (bf16), any batch: 16 tokens per block on warp-level MMAs, W_gate in shared
    // memory, every SM streaming x rows (at a decode batch of 128 tokens, 8 blocks took 11 us
    // against 13 us for one block per token).
    if (bf16 && E == 8 && route_e8_smem(D) <= (size_t)kRouteE8MaxSmem) {
        static std::once_flag once;
        static cudaError_t attr_err = cudaSuccess;
        std::call_once(once, [] {
            attr_err = cudaFuncSetAttribute(route_e8_kernel,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            kRouteE8MaxSmem);
        });
        if (attr_err != cudaSuccess) {
            set_error(MOE_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(attr_err));
            return -1;
        }
        const int64_t blocks = (S + kE8MmaTokens - 1) / kE8MmaTokens;
        route_e8_kernel<<<(unsigned)blocks, kWarps * 32, route_e8_smem(D), s>>>(
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
