// Attention core of Mixture of Attention (ScatterMoE guide, "2. Generalization to Mixture of
// Attention (MoA)"; the ScatterMoE abstract's MoA demonstration). The routed query projection
// leaves q in slot order, one row per (token, selected expert); keys and values are shared by all
// experts, one row per token. For slot p (route i = sorted_rows[p], token s = i / k) and head h:
//   o[p, h] = sum_{t <= s} softmax_t(q[p, h] . K[t, h] / sqrt(dh)) V[t, h]
// i.e. causal attention in which every query row carries its own token position. The output stays
// in slot order for the routed output projection (grouped in, gated scatter-add out).
//
// One block computes 128 slots x one head: 8 warps of 16 query rows, keys in blocks of 64 staged in
// shared memory by cp.async (double buffered, 16-byte pieces, rows XOR-swizzled so that the
// ldmatrix reads are conflict-free). Scores and the output use the tensor cores (mma.sync
// m16n8k16, bf16 operands, fp32 accumulators) with the running-max softmax rescaling of
// FlashAttention: scores never leave registers. A block walks the key blocks up to the largest
// position among its rows; a warp skips key blocks beyond its own rows' positions, and only key
// blocks that reach past a row's position are masked.
#include "moe_internal.cuh"

#include <cuda_bf16.h>
#include <math_constants.h>

#include <climits>
#include <cmath>
#include <mutex>

namespace moe {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kRowsPerWarp = 16;
constexpr int kBlockQ = kWarps * kRowsPerWarp;  // query slots per block
constexpr int kBlockK = 64;                      // keys per step

template <int DH>
struct AttnCfg {
    static constexpr int kRowBytes = DH * 2;
    static constexpr int kChunks = DH / 8;  // 16-byte pieces per row
    static constexpr int kQBytes = kBlockQ * kRowBytes;
    static constexpr int kKVBytes = kBlockK * kRowBytes;
    // Q (reused for the output rows), K[2], V[2], positions
    static constexpr int kSmem = kQBytes + 4 * kKVBytes + kBlockQ * 4 + 64;
};

struct AttnParams {
    const __nv_bfloat16 *q;    // [R, H*dh] slot order
    const __nv_bfloat16 *kv;   // [S, 2*H*dh]: K columns [0, H*dh), V columns [H*dh, 2*H*dh)
    const int32_t *sorted_rows;
    const int32_t *offsets;    // [E+1]: slots at or beyond offsets[E] hold no route
    __nv_bfloat16 *o;          // [R, H*dh] slot order
    int64_t R, S;
    int32_t H, k, E;
    float scale_log2;          // log2(e) / sqrt(dh)
};

// Byte offset of 16-byte piece `c` of row `r` in a swizzled tile.
template <int DH>
__device__ __forceinline__ uint32_t swz(int r, int c) {
    return (uint32_t)(r * AttnCfg<DH>::kRowBytes + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&d)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&d)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
                 : "r"(addr));
}
// D += A . B, m16n8k16, A row-major 16x16 bf16, B column-major 16x8 bf16, fp32 accumulators.
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&v);
}

// Stages `rows` rows of one head (dh columns starting at `col`) from a [*, ld] bf16 matrix into a
// swizzled tile; rows at or past `limit` are zero-filled.
template <int DH>
__device__ __forceinline__ void stage_rows(uint32_t tile, const __nv_bfloat16 *base, int64_t ld,
                                           int64_t col, int64_t row0, int rows, int64_t limit) {
    constexpr int C = AttnCfg<DH>::kChunks;
    for (int i = threadIdx.x; i < rows * C; i += kThreads) {
        const int r = i / C, c = i % C;
        const int64_t gr = row0 + r;
        const bool ok = gr < limit;
        const __nv_bfloat16 *src = ok ? base + gr * ld + col + c * 8 : base;
        dev::cp_async16(tile + swz<DH>(r, c), src, ok ? 16u : 0u);
    }
}

template <int DH>
__global__ void __launch_bounds__(kThreads, 1) moa_attention_kernel(AttnParams p) {
    using Cfg = AttnCfg<DH>;
    constexpr int KS = DH / 16;  // k-steps over the head dimension
    constexpr int ND = DH / 8;   // n-tiles of the output
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t sQ = dev::smem_u32(smem);
    const uint32_t sK = sQ + Cfg::kQBytes;
    const uint32_t sV = sK + 2 * Cfg::kKVBytes;
    int *pos = reinterpret_cast<int *>(smem + Cfg::kQBytes + 4 * Cfg::kKVBytes);
    int *wmax = pos + kBlockQ;

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int64_t tile = blockIdx.x / p.H;
    const int h = blockIdx.x % p.H;
    const int64_t HD = (int64_t)p.H * DH;
    const int64_t p0 = tile * kBlockQ;
    const int64_t r_valid = min(p.R, (int64_t)__ldg(p.offsets + p.E));

    if (threadIdx.x < kBlockQ) {
        const int64_t slot = p0 + threadIdx.x;
        int ps = -1;
        if (slot < r_valid) {
            const int32_t route = __ldg(p.sorted_rows + slot);
            if (route >= 0 && route < p.R) ps = route / p.k;
        }
        pos[threadIdx.x] = ps;
    }
    __syncthreads();
    // this warp's rows: positions of rows g and g + 8 for this lane's quad
    const int g = lane >> 2, t4 = lane & 3;
    const int pos0 = pos[warp * 16 + g], pos1 = pos[warp * 16 + g + 8];
    int wlo = lane < 16 ? pos[warp * 16 + lane] : INT_MAX;
    int whi = lane < 16 ? pos[warp * 16 + lane] : -1;
    for (int off = 16; off > 0; off >>= 1) {
        wlo = min(wlo, __shfl_xor_sync(0xffffffffu, wlo, off));
        whi = max(whi, __shfl_xor_sync(0xffffffffu, whi, off));
    }
    if (lane == 0) wmax[warp] = whi;
    __syncthreads();
    int bmax = -1;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) bmax = max(bmax, wmax[w]);
    if (bmax < 0) return;  // no route in this tile (uniform over the block)
    const int nkb = bmax / kBlockK + 1;

    stage_rows<DH>(sQ, p.q, HD, (int64_t)h * DH, p0, kBlockQ, r_valid);
    stage_rows<DH>(sK, p.kv, 2 * HD, (int64_t)h * DH, 0, kBlockK, p.S);
    stage_rows<DH>(sV, p.kv, 2 * HD, HD + (int64_t)h * DH, 0, kBlockK, p.S);
    dev::cp_async_commit_group();

    uint32_t qf[KS][4];
    float oacc[ND][4];
#pragma unroll
    for (int n = 0; n < ND; ++n) oacc[n][0] = oacc[n][1] = oacc[n][2] = oacc[n][3] = 0.f;
    float m0 = -CUDART_INF_F, m1 = -CUDART_INF_F, l0 = 0.f, l1 = 0.f;
    const int mi = lane >> 3, mr = lane & 7;  // ldmatrix: this lane addresses row mr of matrix mi

    for (int j = 0; j < nkb; ++j) {
        const int buf = j & 1;
        if (j + 1 < nkb) {
            const uint32_t nb = (uint32_t)((j + 1) & 1) * Cfg::kKVBytes;
            stage_rows<DH>(sK + nb, p.kv, 2 * HD, (int64_t)h * DH, (int64_t)(j + 1) * kBlockK,
                           kBlockK, p.S);
            stage_rows<DH>(sV + nb, p.kv, 2 * HD, HD + (int64_t)h * DH,
                           (int64_t)(j + 1) * kBlockK, kBlockK, p.S);
        }
        dev::cp_async_commit_group();
        dev::cp_async_wait_group<1>();
        __syncthreads();
        if (j == 0) {
#pragma unroll
            for (int kk = 0; kk < KS; ++kk)
                ldsm_x4(sQ + swz<DH>(warp * 16 + (mi & 1) * 8 + mr, 2 * kk + (mi >> 1)), qf[kk]);
        }
        const int key0 = j * kBlockK;
        if (key0 <= whi) {
            const uint32_t tK = sK + buf * Cfg::kKVBytes, tV = sV + buf * Cfg::kKVBytes;
            float sacc[kBlockK / 8][4];
#pragma unroll
            for (int n = 0; n < kBlockK / 8; ++n) sacc[n][0] = sacc[n][1] = sacc[n][2] = sacc[n][3] = 0.f;
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) {
#pragma unroll
                for (int np = 0; np < kBlockK / 16; ++np) {
                    uint32_t b[4];
                    ldsm_x4(tK + swz<DH>(np * 16 + (mi >> 1) * 8 + mr, 2 * kk + (mi & 1)), b);
                    mma16816(sacc[2 * np], qf[kk], b[0], b[1]);
                    mma16816(sacc[2 * np + 1], qf[kk], b[2], b[3]);
                }
            }
            // scale into the log2 domain; mask keys past each row's position
            const bool need_mask = key0 + kBlockK - 1 > wlo;
            float mx0 = -CUDART_INF_F, mx1 = -CUDART_INF_F;
#pragma unroll
            for (int n = 0; n < kBlockK / 8; ++n) {
                const int t = key0 + n * 8 + 2 * t4;
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    float s0 = sacc[n][e] * p.scale_log2, s1 = sacc[n][2 + e] * p.scale_log2;
                    if (need_mask) {
                        if (t + e > pos0) s0 = -CUDART_INF_F;
                        if (t + e > pos1) s1 = -CUDART_INF_F;
                    }
                    sacc[n][e] = s0;
                    sacc[n][2 + e] = s1;
                    mx0 = fmaxf(mx0, s0);
                    mx1 = fmaxf(mx1, s1);
                }
            }
#pragma unroll
            for (int off = 1; off <= 2; off <<= 1) {
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
            }
            const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
            // a row with every key so far masked keeps m = -inf; subtract 0 instead (all p are 0)
            const float u0 = n0 == -CUDART_INF_F ? 0.f : n0, u1 = n1 == -CUDART_INF_F ? 0.f : n1;
            const float a0 = exp2f(m0 - u0), a1 = exp2f(m1 - u1);
            m0 = n0;
            m1 = n1;
            float s0sum = 0.f, s1sum = 0.f;
#pragma unroll
            for (int n = 0; n < kBlockK / 8; ++n) {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    sacc[n][e] = exp2f(sacc[n][e] - u0);
                    sacc[n][2 + e] = exp2f(sacc[n][2 + e] - u1);
                    s0sum += sacc[n][e];
                    s1sum += sacc[n][2 + e];
                }
            }
            l0 = l0 * a0 + s0sum;
            l1 = l1 * a1 + s1sum;
#pragma unroll
            for (int n = 0; n < ND; ++n) {
                oacc[n][0] *= a0;
                oacc[n][1] *= a0;
                oacc[n][2] *= a1;
                oacc[n][3] *= a1;
            }
#pragma unroll
            for (int kk = 0; kk < kBlockK / 16; ++kk) {
                const uint32_t a[4] = {pack_bf16(sacc[2 * kk][0], sacc[2 * kk][1]),
                                       pack_bf16(sacc[2 * kk][2], sacc[2 * kk][3]),
                                       pack_bf16(sacc[2 * kk + 1][0], sacc[2 * kk + 1][1]),
                                       pack_bf16(sacc[2 * kk + 1][2], sacc[2 * kk + 1][3])};
#pragma unroll
                for (int dp = 0; dp < DH / 16; ++dp) {
                    uint32_t b[4];
                    ldsm_x4_t(tV + swz<DH>(kk * 16 + (mi & 1) * 8 + mr, 2 * dp + (mi >> 1)), b);
                    mma16816(oacc[2 * dp], a, b[0], b[1]);
                    mma16816(oacc[2 * dp + 1], a, b[2], b[3]);
                }
            }
        }
        __syncthreads();  // the next iteration refills this buffer
    }

    // normalise; stage this warp's 16 rows in its own rows of the Q tile, then 16-byte stores
#pragma unroll
    for (int off = 1; off <= 2; off <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, off);
        l1 += __shfl_xor_sync(0xffffffffu, l1, off);
    }
    const float i0 = l0 > 0.f ? 1.f / l0 : 0.f, i1 = l1 > 0.f ? 1.f / l1 : 0.f;
#pragma unroll
    for (int n = 0; n < ND; ++n) {
        const int c = n * 8 + 2 * t4;  // column inside the head
        const uint32_t r0 = sQ + swz<DH>(warp * 16 + g, c / 8) + (c % 8) * 2;
        const uint32_t r1 = sQ + swz<DH>(warp * 16 + g + 8, c / 8) + (c % 8) * 2;
        asm volatile("st.shared.b32 [%0], %1;" ::"r"(r0), "r"(pack_bf16(oacc[n][0] * i0, oacc[n][1] * i0)));
        asm volatile("st.shared.b32 [%0], %1;" ::"r"(r1), "r"(pack_bf16(oacc[n][2] * i1, oacc[n][3] * i1)));
    }
    __syncwarp();
    constexpr int C = Cfg::kChunks;
    for (int i = lane; i < 16 * C; i += 32) {
        const int r = i / C, c = i % C;
        const int64_t slot = p0 + warp * 16 + r;
        if (slot >= r_valid) continue;
        uint4 v;
        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                     : "r"(sQ + swz<DH>(warp * 16 + r, c)));
        *reinterpret_cast<uint4 *>(p.o + slot * HD + (int64_t)h * DH + c * 8) = v;
    }
}

template <int DH>
int launch_dh(const AttnParams &p, cudaStream_t s) {
    constexpr int smem = AttnCfg<DH>::kSmem;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [&] {
        attr_err = cudaFuncSetAttribute(moa_attention_kernel<DH>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    });
    if (attr_err != cudaSuccess)
        return set_error(MOE_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(attr_err));
    const int64_t tiles = (p.R + kBlockQ - 1) / kBlockQ;
    const int64_t blocks = tiles * p.H;
    if (blocks > 0x7fffffffLL) return set_error(MOE_ERR_INVALID_ARG, "moa attention: grid too large");
    moa_attention_kernel<DH><<<(unsigned)blocks, kThreads, smem, s>>>(p);
    return MOE_OK;
}

}  // namespace

int launch_moa_attention(const void *q, const void *kv, const int32_t *sorted_rows,
                         const int32_t *offsets, void *o, int64_t R, int64_t S, int32_t H,
                         int32_t dh, int32_t k, int32_t E, cudaStream_t s) {
    if (R == 0) return MOE_OK;
    AttnParams p;
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.kv = static_cast<const __nv_bfloat16 *>(kv);
    p.sorted_rows = sorted_rows;
    p.offsets = offsets;
    p.o = static_cast<__nv_bfloat16 *>(o);
    p.R = R;
    p.S = S;
    p.H = H;
    p.k = k;
    p.E = E;
    p.scale_log2 = (float)(1.4426950408889634 / sqrt((double)dh));
    if (dh == 128) return launch_dh<128>(p, s);
    if (dh == 64) return launch_dh<64>(p, s);
    return set_error(MOE_ERR_UNSUPPORTED, "moa attention: head size %d (64 or 128 are built)", dh);
}

// The single-group offsets {0, S} of the shared key/value projection (one "expert" holding every
// token).
__global__ void kv_offsets_kernel(int32_t *off, int32_t S) {
    if (threadIdx.x == 0) {
        off[0] = 0;
        off[1] = S;
    }
}

void launch_kv_offsets(int32_t *off, int64_t S, cudaStream_t s) {
    kv_offsets_kernel<<<1, 32, 0, s>>>(off, (int32_t)S);
}

}  // namespace moe
