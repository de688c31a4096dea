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

// =============================================================================================
// tcgen05 attention core
// =============================================================================================
// Query rows in route order: tile t holds routes [128 t, 128 t + 128), i.e. the k routes of 128/k
// consecutive tokens, so a tile's rows share nearly one causal limit and the cost of a tile grows
// with t. Row i reads q from slot sparse_rows[i] and writes o there. Work items are (tile, head)
// in order of decreasing tile; persistent CTAs take every gridDim.x-th item.
//
// Roles (192 threads): warp 0 loads K and V blocks of 128 keys by TMA (two stages); warp 1 issues
// the MMAs: S = Q K^T into one of two TMEM score buffers, then O += P V into the TMEM output;
// warps 2-5 own one query row per thread (= TMEM lane): they read the score row, mask keys past
// the row's token, keep a reference maximum that moves only when the row maximum exceeds it by
// more than 2^8 (scores stay exact, exponentials stay below 256), write the bf16 probabilities P
// into shared memory as the next MMA's A operand (128-byte swizzle), and rescale O in TMEM when
// a row's reference moved. The last P V of a tile leaves O complete: they normalise by the row
// sum and store bf16 rows to the slots. Q of the next tile is gathered by cp.async (one row per
// thread) as soon as the last score MMA of the current tile has completed.
namespace tc {

constexpr int BM = 128;                  // query rows per tile
constexpr int BN = 128;                  // keys per block
constexpr int THREADS = 192;
constexpr uint32_t CHUNK = 128u * 128u;  // 128 rows x 128 bytes, swizzled
constexpr uint32_t TMEM_COLS = 512;      // S[0] at 0, S[1] at 128, O at 256
constexpr uint32_t O_COL = 256;
constexpr float kRescaleLog2 = 8.0f;

template <int DH>
struct Layout {
    static constexpr int NCH = DH / 64;
    static constexpr uint32_t Q = NCH * CHUNK;
    static constexpr uint32_t KV = NCH * CHUNK;
    static constexpr uint32_t P = (BN / 64) * CHUNK;
    static constexpr uint32_t OFF_K = Q;
    static constexpr uint32_t OFF_V = OFF_K + 2 * KV;
    static constexpr uint32_t OFF_P = OFF_V + 2 * KV;
    static constexpr uint32_t OFF_BAR = OFF_P + 2 * P;
    static constexpr uint32_t SMEM = OFF_BAR + 256 + 1024;  // + barriers + alignment slack
    static constexpr uint32_t TX = 2 * KV;                  // K and V bytes of one block
};

struct Bars {
    uint64_t kv_full[2], kv_empty[2], s_full[2], s_free[2], p_full[2], p_empty[2];
    uint64_t q_full, o_free, drain;
    uint32_t tmem_base;
    int abort;
};

struct Params {
    const __nv_bfloat16 *q;       // [R, HD] slot order
    const int32_t *sparse_rows;   // [R] route -> slot (negative: no slot)
    __nv_bfloat16 *o;             // [R, HD] slot order
    int64_t R, S, nitems;
    int32_t H, k, ntiles;
    float scale_log2;
    unsigned *status;
    int64_t wait_limit_ns;
};

// Byte offset of 16-byte unit u (8 bf16) of row r in a K-major tile of 128 rows with 128-byte
// swizzle: 64-column chunks of CHUNK bytes, 8-row atoms of 1024 bytes.
__device__ __forceinline__ uint32_t sw_off(int r, int u) {
    return (uint32_t)(u >> 3) * CHUNK + (uint32_t)(r >> 3) * 1024u + (uint32_t)(r & 7) * 128u +
           ((uint32_t)((u & 7) ^ (r & 7)) << 4);
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

template <int DH>
__global__ void __launch_bounds__(THREADS, 1)
moa_attention_tc_kernel(const __grid_constant__ CUtensorMap tmKV, const Params p) {
    using L = Layout<DH>;
    constexpr uint32_t IDESC_S = dev::idesc_f32acc(true, BM, BN, false);
    constexpr uint32_t IDESC_O = dev::idesc_f32acc(true, BM, DH, true);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = dev::smem_u32(smem);
    Bars &bar = *reinterpret_cast<Bars *>(smem + L::OFF_BAR);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t HD = (int64_t)p.H * DH;

    if (threadIdx.x == 0) {
        for (int b = 0; b < 2; ++b) {
            dev::mbar_init(&bar.kv_full[b], 1);
            dev::mbar_init(&bar.kv_empty[b], 1);
            dev::mbar_init(&bar.s_full[b], 1);
            dev::mbar_init(&bar.s_free[b], BM);
            dev::mbar_init(&bar.p_full[b], BM);
            dev::mbar_init(&bar.p_empty[b], 1);
        }
        dev::mbar_init(&bar.q_full, BM);
        dev::mbar_init(&bar.o_free, BM);
        dev::mbar_init(&bar.drain, 1);
        bar.abort = 0;
        dev::fence_mbar_init();
    }
    if (warp == 0 && lane == 0) dev::prefetch_tmap(&tmKV);
    if (warp == 1) {
        dev::tmem_alloc(&bar.tmem_base, TMEM_COLS);
        dev::tmem_relinquish();
        dev::tc_fence_before();
    }
    __syncthreads();
    dev::tc_fence_after();
    const uint32_t tmem = bar.tmem_base;
    volatile int *abort = &bar.abort;
    // item -> (tile, head); blocks of 128 keys the tile needs (up to its last token)
    auto tile_of = [&](int64_t it) { return (int64_t)p.ntiles - 1 - it / p.H; };
    auto head_of = [&](int64_t it) { return (int)(it % p.H); };
    auto nblocks = [&](int64_t tile) {
        const int64_t last = min(p.R, (tile + 1) * BM) - 1;
        return (int)((last / p.k) / BN) + 1;
    };

    if (warp == 0) {
        // ---------------------------------------------------------------- K/V producer
        if (lane == 0) {
            uint32_t g = 0, issued = 0, last_par = 0;
            bool ok = true;
            for (int64_t it = blockIdx.x; it < p.nitems && ok; it += gridDim.x) {
                const int64_t tile = tile_of(it);
                const int h = head_of(it);
                const int n = nblocks(tile);
                for (int j = 0; j < n; ++j, ++g) {
                    const uint32_t b = g & 1u;
                    if (g >= 2 && !dev::mbar_wait(&bar.kv_empty[b], ((g - 2) >> 1) & 1u, abort,
                                                  p.status, p.wait_limit_ns, kKernelAttention)) {
                        ok = false;
                        break;
                    }
                    dev::mbar_arrive_expect_tx(&bar.kv_full[b], L::TX);
#pragma unroll
                    for (int c = 0; c < L::NCH; ++c) {
                        dev::tma_load_2d(smem + L::OFF_K + b * L::KV + c * CHUNK, &tmKV,
                                         &bar.kv_full[b], (int32_t)(h * DH + c * 64),
                                         (int32_t)(j * BN));
                        dev::tma_load_2d(smem + L::OFF_V + b * L::KV + c * CHUNK, &tmKV,
                                         &bar.kv_full[b], (int32_t)(HD + h * DH + c * 64),
                                         (int32_t)(j * BN));
                    }
                    issued |= 1u << b;
                    last_par = (last_par & ~(1u << b)) | (((g >> 1) & 1u) << b);
                }
            }
            // teardown: every load issued must land before the CTA may exit
            for (int b = 0; b < 2; ++b)
                if (issued & (1u << b))
                    dev::mbar_wait(&bar.kv_full[b], (last_par >> b) & 1u, nullptr, p.status,
                                   kDrainLimitNs, kKernelAttention);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            auto wait = [&](uint64_t *b, uint32_t par) {
                return dev::mbar_wait(b, par, abort, p.status, p.wait_limit_ns, kKernelAttention);
            };
            // O += P V for global block gp (the first block of a tile overwrites O, after the
            // softmax warps have read the previous tile's O)
            auto pv = [&](uint32_t gp, bool first, uint32_t tcnt) {
                const uint32_t b = gp & 1u;
                if (!wait(&bar.p_full[b], (gp >> 1) & 1u)) return false;
                if (first && tcnt > 0 && !wait(&bar.o_free, (tcnt - 1) & 1u)) return false;
                dev::tc_fence_after();
                const uint32_t sP = sbase + L::OFF_P + b * L::P;
                const uint32_t sV = sbase + L::OFF_V + b * L::KV;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    const uint64_t ad =
                        dev::sdesc(sP + (kk >> 2) * CHUNK + (kk & 3) * 32, 16, 1024, dev::kLayoutSw128);
                    const uint64_t bd = dev::sdesc(sV + kk * 2048, CHUNK, 1024, dev::kLayoutSw128);
                    dev::mma_bf16(tmem + O_COL, ad, bd, IDESC_O, (!first || kk > 0) ? 1u : 0u);
                }
                dev::mma_commit(&bar.p_empty[b]);
                dev::mma_commit(&bar.kv_empty[b]);
                return true;
            };
            uint32_t g = 0, tcnt = 0;
            bool ok = true;
            for (int64_t it = blockIdx.x; it < p.nitems && ok; it += gridDim.x, ++tcnt) {
                const int n = nblocks(tile_of(it));
                if (!wait(&bar.q_full, tcnt & 1u)) break;
                for (int j = 0; j < n; ++j) {
                    const uint32_t gj = g + j, b = gj & 1u;
                    if (!wait(&bar.kv_full[b], (gj >> 1) & 1u) ||
                        (gj >= 2 && !wait(&bar.s_free[b], ((gj - 2) >> 1) & 1u))) {
                        ok = false;
                        break;
                    }
                    dev::tc_fence_after();
                    const uint32_t sK = sbase + L::OFF_K + b * L::KV;
#pragma unroll
                    for (int kk = 0; kk < DH / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * CHUNK + (kk & 3) * 32;
                        dev::mma_bf16(tmem + b * BN,
                                      dev::sdesc(sbase + off, 16, 1024, dev::kLayoutSw128),
                                      dev::sdesc(sK + off, 16, 1024, dev::kLayoutSw128), IDESC_S,
                                      kk > 0 ? 1u : 0u);
                    }
                    dev::mma_commit(&bar.s_full[b]);
                    if (j >= 1 && !pv(gj - 1, j == 1, tcnt)) {
                        ok = false;
                        break;
                    }
                }
                if (!ok || !pv(g + n - 1, n == 1, tcnt)) break;
                g += n;
            }
            // teardown: all issued MMAs complete before TMEM is released
            dev::mma_commit(&bar.drain);
            dev::mbar_wait(&bar.drain, 0, nullptr, p.status, kDrainLimitNs, kKernelAttention);
            dev::tc_fence_before();
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- softmax warps
        const int qw = warp & 3;            // TMEM lane quarter this warp may access
        const int row = qw * 32 + lane;     // query row of the tile = TMEM lane
        const uint32_t tl = tmem + ((uint32_t)(qw * 32) << 16);
        auto wait = [&](uint64_t *b, uint32_t par) {  // warp-uniform bounded wait
            bool w = true;
            if (lane == 0)
                w = dev::mbar_wait(b, par, abort, p.status, p.wait_limit_ns, kKernelAttention);
            return __shfl_sync(0xffffffffu, w, 0) != 0;
        };
        auto slot_of = [&](int64_t tile) {
            const int64_t i = tile * BM + row;
            const int32_t sl = i < p.R ? __ldg(p.sparse_rows + i) : -1;
            return (sl >= 0 && sl < p.R) ? (int64_t)sl : (int64_t)-1;
        };
        // this thread's row of Q for (tile, head) -> the Q tile (zeros without a slot)
        auto load_q = [&](int64_t tile, int h) {
            const int64_t sl = slot_of(tile);
            const __nv_bfloat16 *src = sl >= 0 ? p.q + sl * HD + (int64_t)h * DH : p.q;
#pragma unroll
            for (int u = 0; u < DH / 8; ++u)
                dev::cp_async16(sbase + sw_off(row, u), sl >= 0 ? src + u * 8 : p.q,
                                sl >= 0 ? 16u : 0u);
        };
        uint32_t g = 0;
        bool ok = true;
        if ((int64_t)blockIdx.x < p.nitems) {
            load_q(tile_of(blockIdx.x), head_of(blockIdx.x));
            dev::cp_async_wait_all();
            dev::fence_proxy_async_smem();
            dev::mbar_arrive(&bar.q_full);
        }
        for (int64_t it = blockIdx.x; it < p.nitems && ok; it += gridDim.x) {
            const int64_t tile = tile_of(it);
            const int h = head_of(it);
            const int n = nblocks(tile);
            const int64_t slot = slot_of(tile);
            const int pos = slot >= 0 ? (int)((tile * BM + row) / p.k) : -1;
            const bool has_next = it + gridDim.x < p.nitems;
            float m_ref = -CUDART_INF_F, l = 0.f;
            for (int j = 0; j < n && ok; ++j) {
                const uint32_t gj = g + j, b = gj & 1u;
                if (!wait(&bar.s_full[b], (gj >> 1) & 1u)) {
                    ok = false;
                    break;
                }
                dev::tc_fence_after();
                uint32_t sr[BN / 32][32];
#pragma unroll
                for (int c = 0; c < BN / 32; ++c) dev::tmem_ld32(tl + b * BN + c * 32, sr[c]);
                dev::tmem_ld_wait();
                dev::tc_fence_before();
                dev::mbar_arrive(&bar.s_free[b]);
                // the last score MMA of this tile has completed: Q may be replaced
                if (j == n - 1 && has_next) load_q(tile_of(it + gridDim.x), head_of(it + gridDim.x));
                const int key0 = j * BN;
                if (key0 + BN - 1 > pos) {
#pragma unroll
                    for (int c = 0; c < BN; ++c)
                        if (key0 + c > pos) sr[c / 32][c % 32] = __float_as_uint(-CUDART_INF_F);
                }
                float mx = -CUDART_INF_F;
#pragma unroll
                for (int c = 0; c < BN; ++c) mx = fmaxf(mx, __uint_as_float(sr[c / 32][c % 32]));
                const float mxs = mx * p.scale_log2;
                const bool need = mxs > m_ref + kRescaleLog2;
                float alpha = 1.f;
                if (need) {
                    alpha = ex2(m_ref - mxs);
                    m_ref = mxs;
                }
                const float mneg = m_ref == -CUDART_INF_F ? 0.f : -m_ref;
                // P row (bf16) into P buffer b once P V of block gj - 2 has released it
                if (gj >= 2 && !wait(&bar.p_empty[b], ((gj - 2) >> 1) & 1u)) {
                    ok = false;
                    break;
                }
                const uint32_t sP = sbase + L::OFF_P + b * L::P;
                float sum = 0.f;
#pragma unroll
                for (int u = 0; u < BN / 8; ++u) {
                    float e[8];
#pragma unroll
                    for (int t = 0; t < 8; ++t) {
                        e[t] = ex2(fmaf(__uint_as_float(sr[(u * 8 + t) / 32][(u * 8 + t) % 32]),
                                        p.scale_log2, mneg));
                        sum += e[t];
                    }
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(sP + sw_off(row, u)),
                                 "r"(pack_bf16(e[0], e[1])), "r"(pack_bf16(e[2], e[3])),
                                 "r"(pack_bf16(e[4], e[5])), "r"(pack_bf16(e[6], e[7]))
                                 : "memory");
                }
                l = l * alpha + sum;
                dev::fence_proxy_async_smem();
                // O holds P V of blocks < gj: rescale the rows whose reference moved
                if (j >= 1 && __any_sync(0xffffffffu, need)) {
                    const uint32_t gp = gj - 1;
                    if (!wait(&bar.p_empty[gp & 1u], (gp >> 1) & 1u)) {
                        ok = false;
                        break;
                    }
                    dev::tc_fence_after();
#pragma unroll
                    for (int c = 0; c < DH / 32; ++c) {
                        uint32_t o[32];
                        dev::tmem_ld32(tl + O_COL + c * 32, o);
                        dev::tmem_ld_wait();
#pragma unroll
                        for (int t = 0; t < 32; ++t) o[t] = __float_as_uint(__uint_as_float(o[t]) * alpha);
                        dev::tmem_st32(tl + O_COL + c * 32, o);
                    }
                    dev::tmem_st_wait();
                }
                dev::tc_fence_before();
                dev::mbar_arrive(&bar.p_full[b]);
            }
            if (!ok) break;
            // O complete after P V of the tile's last block: normalise and store the row
            const uint32_t gl = g + n - 1;
            if (!wait(&bar.p_empty[gl & 1u], (gl >> 1) & 1u)) break;
            dev::tc_fence_after();
            const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
            for (int c = 0; c < DH / 32; ++c) {
                uint32_t o[32];
                dev::tmem_ld32(tl + O_COL + c * 32, o);
                dev::tmem_ld_wait();
                if (slot >= 0) {
                    uint4 *dst = reinterpret_cast<uint4 *>(p.o + slot * HD + (int64_t)h * DH + c * 32);
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        uint4 w;
                        w.x = pack_bf16(__uint_as_float(o[8 * v + 0]) * inv, __uint_as_float(o[8 * v + 1]) * inv);
                        w.y = pack_bf16(__uint_as_float(o[8 * v + 2]) * inv, __uint_as_float(o[8 * v + 3]) * inv);
                        w.z = pack_bf16(__uint_as_float(o[8 * v + 4]) * inv, __uint_as_float(o[8 * v + 5]) * inv);
                        w.w = pack_bf16(__uint_as_float(o[8 * v + 6]) * inv, __uint_as_float(o[8 * v + 7]) * inv);
                        dst[v] = w;
                    }
                }
            }
            dev::tc_fence_before();
            dev::mbar_arrive(&bar.o_free);
            if (has_next) {
                dev::cp_async_wait_all();
                dev::fence_proxy_async_smem();
                dev::mbar_arrive(&bar.q_full);
            }
            g += n;
        }
        dev::cp_async_wait_all();  // no copy into this CTA's shared memory outlives it
    }
    __syncthreads();
    if (warp == 1) {
        dev::tc_fence_after();
        dev::tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace tc

template <int DH>
int launch_tc(const void *q, const void *kv, const int32_t *sparse_rows, void *o, int64_t R,
              int64_t S, int32_t H, int32_t k, unsigned *status, cudaStream_t s) {
    using L = tc::Layout<DH>;
    auto kern = tc::moa_attention_tc_kernel<DH>;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [&] {
        attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)L::SMEM);
    });
    if (attr_err != cudaSuccess)
        return set_error(MOE_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(attr_err));
    const int64_t HD = (int64_t)H * DH;
    CUtensorMap m;
    const uint64_t dims[2] = {(uint64_t)(2 * HD), (uint64_t)S};
    const uint64_t str[1] = {(uint64_t)(2 * HD) * 2};
    const uint32_t box[2] = {64, (uint32_t)tc::BN};
    int rc = encode_tmap(&m, true, 2, kv, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
    tc::Params p;
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.sparse_rows = sparse_rows;
    p.o = static_cast<__nv_bfloat16 *>(o);
    p.R = R;
    p.S = S;
    p.H = H;
    p.k = k;
    p.ntiles = (int32_t)((R + tc::BM - 1) / tc::BM);
    p.nitems = (int64_t)p.ntiles * H;
    p.scale_log2 = (float)(1.4426950408889634 / sqrt((double)DH));
    p.status = status;
    p.wait_limit_ns = kWaitLimitNs;
    const int grid = (int)std::min<int64_t>(num_sms(), p.nitems);
    kern<<<grid, tc::THREADS, L::SMEM, s>>>(m, p);
    return MOE_OK;
}

}  // namespace

int launch_moa_attention(const void *q, const void *kv, const int32_t *sorted_rows,
                         const int32_t *sparse_rows, const int32_t *offsets, void *o, int64_t R,
                         int64_t S, int32_t H, int32_t dh, int32_t k, int32_t E, unsigned *status,
                         cudaStream_t s) {
    if (R == 0) return MOE_OK;
    if (dh != 64 && dh != 128)
        return set_error(MOE_ERR_UNSUPPORTED, "moa attention: head size %d (64 or 128 are built)", dh);
    if (R >= (int64_t(1) << 31) - tc::BM || S >= (int64_t(1) << 31) - tc::BN)
        return set_error(MOE_ERR_INVALID_ARG, "moa attention: sizes too large");
    const char *legacy = getenv("MOE_ATTN_MMA_SYNC");
    if (legacy == nullptr || legacy[0] != '1')
        return dh == 128 ? launch_tc<128>(q, kv, sparse_rows, o, R, S, H, k, status, s)
                         : launch_tc<64>(q, kv, sparse_rows, o, R, S, H, k, status, s);
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
    return dh == 128 ? launch_dh<128>(p, s) : launch_dh<64>(p, s);
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
