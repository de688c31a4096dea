// Pieces shared by the one-CTA and the two-CTA (cta_group::2) grouped GEMM kernels: tile
// constants, kernel parameters, the device-side tile schedule and the per-row epilogue.
#pragma once

#include "moe_internal.cuh"

namespace moe {
namespace gemm {

constexpr int BM = 128;                 // rows per tile (TMEM lanes)
constexpr int BN = 256;                 // MMA N = accumulator columns
constexpr int STAGES = 4;
constexpr int MAX_STAGES = 8;           // router mode: up to 8 smaller stages in the same space
constexpr size_t STAGE_AREA = (size_t)STAGES * (128 * 128 + 256 * 128);
constexpr int KBYTES = 128;             // bytes of K per stage (one 128-byte swizzle row)
constexpr int A_BYTES = BM * KBYTES;    // 16 KB
constexpr int B_BYTES = BN * KBYTES;    // 32 KB (BN columns x (128 / eb) K rows x eb)
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int MAX_E = 256;
constexpr int THREADS = 192;            // producer, MMA, 4 epilogue warps
constexpr int GATHER_THREADS = 128;     // extra warps 6-9 for gathered A
constexpr uint32_t TMEM_COLS = 512;

// Shared-memory bookkeeping of the one-CTA kernel (after its STAGES operand stages).
struct SmemTail {
    uint64_t full[MAX_STAGES];
    uint64_t empty[MAX_STAGES];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    int32_t off[MAX_E + 1];
    int32_t tstart[MAX_E + 1];
    float stage[4][32 * 33];  // per epilogue warp: 32 rows x 32 columns (+1 pad) of one chunk
};
constexpr size_t SMEM_BYTES = 1024 + STAGE_AREA + sizeof(SmemTail);

struct KParams {
    const void *A;    // gathered mode: x [S, K] (rows fetched by the gather warps)
    int64_t K;
    const int32_t *offsets;
    const int32_t *sorted_rows;
    const float *gates;
    void *out;
    int32_t E, k;
    int32_t N;        // output columns
    int32_t num_kb;   // K stages
    int32_t n_tiles;  // N tiles
    int64_t S, R;     // bounds of scatter rows (tokens) and grouped rows (slots)
    // router mode: logit bias [E] (nullable), outputs [S, k]
    const float *bias;
    int32_t *top_e;
    float *top_w;
    int32_t b_chunks; // B chunks loaded per stage (router: ceil(E / chunk width))
    int32_t stages;   // router mode: pipeline depth and stage size (bytes, multiple of 1024)
    int32_t stage_bytes;
    int32_t k_split;  // K-major B: first K index read from the second B tensor map
    int32_t a_row_pad;  // contiguous A: slot row p of expert e is read at row p + a_row_pad * e
    // GLU backward epilogue (the MLP backward's recompute of GEMM1): the ungated gradient of h
    // [R, N] bf16 in slot order, the route-weight gradient [R] (accumulated), the output row pad
    const void *bwd_dh;
    float *bwd_dw;
    int32_t out_row_pad;
    // optional side job of the epilogue warps before their first tile: zero zero_n4 float4s
    float4 *zero_ptr;
    int64_t zero_n4;
    unsigned *status;
    int64_t wait_limit_ns;
};

struct TileInfo {
    int e, row_begin, rows, n_idx;
};

// Device-side tile schedule. Expert e owns ceil(N_e / TM) M tiles of TM rows (the last one
// partial, none for an empty expert) times n_tiles N tiles; tstart[e] is the exclusive prefix of
// those counts over experts. Tiles are numbered expert-major, then N tile, then M tile, so the
// CTAs that run at the same time share one expert's weight tiles and gathered rows in L2.
template <int TM>
__device__ __forceinline__ void build_schedule(const int32_t *off, int32_t *tstart, int E,
                                               int n_tiles) {
    int run = 0;
    for (int e = 0; e < E; ++e) {
        tstart[e] = run;
        run += ((off[e + 1] - off[e] + TM - 1) / TM) * n_tiles;
    }
    tstart[E] = run;
}

// Debug builds: the expert offsets behind a schedule must start at 0 or above, never decrease and
// end at or below the slot count R; otherwise the status word records kStatusBadIndex and the
// schedule is emptied (no tile reads a slot index derived from them). Release builds trust the
// offsets, which the sparse map produced.
__device__ __forceinline__ void debug_check_offsets(const int32_t *off, int32_t *tstart, int E,
                                                    int64_t R, unsigned *status) {
    if constexpr (kDebugChecks) {
        bool ok = off[0] >= 0 && (int64_t)off[E] <= R;
        for (int e = 0; e < E; ++e) ok = ok && off[e] <= off[e + 1];
        if (!ok) {
            if (status != nullptr) atomicOr(status, kStatusBadIndex);
            for (int e = 0; e <= E; ++e) tstart[e] = 0;
        }
    }
}

template <int TM>
__device__ __forceinline__ TileInfo decode_tile(int t, const int32_t *off, const int32_t *tstart,
                                                int E) {
    int lo = 0, hi = E;  // tstart[lo] <= t < tstart[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (tstart[mid] <= t) lo = mid;
        else hi = mid;
    }
    TileInfo ti;
    ti.e = lo;
    const int local = t - tstart[lo];
    const int cnt = off[lo + 1] - off[lo];
    const int mt = (cnt + TM - 1) / TM;
    ti.n_idx = local / mt;
    const int m = local - ti.n_idx * mt;
    ti.row_begin = off[lo] + m * TM;
    ti.rows = min(TM, off[lo + 1] - ti.row_begin);
    return ti;
}

__device__ __forceinline__ float silu_f(float z) { return z / (1.0f + __expf(-z)); }


// Epilogue of one accumulator row (the calling thread's TMEM lane) of a 128 x 256 tile:
//   GLU:      h = silu(acc[:, c]) * acc[:, 128 + c] (* g), rounded to the output dtype, stored
//             at out[orow, n0 + c] for the 128 output columns c;
//   SCATTER:  out[orow, n0 + c] += g * acc[:, c] with fp32 vector atomics (256 columns),
//             through the warp's `stage` buffer (32 x 33 floats of shared memory);
//   else:     out[orow, n0 + c] = g * acc[:, c] in the output dtype (256 columns).
// Columns at or past N are skipped (N is a multiple of 8). `valid` is false for rows past the
// tile's end; every lane of the warp calls this together (warp-wide TMEM loads and shuffles).
// The epilogue warps are idle until the first accumulator of the CTA is ready; the MoE forward
// has them zero its fp32 output there (GEMM2 scatter-adds into it only after GEMM1 has ended).
__device__ __forceinline__ void zero_side_job(const KParams &p, int epi_thread, int epi_threads) {
    if (p.zero_ptr == nullptr) return;
    const int64_t stride = (int64_t)gridDim.x * epi_threads;
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int64_t i = (int64_t)blockIdx.x * epi_threads + epi_thread; i < p.zero_n4; i += stride)
        p.zero_ptr[i] = z;
}

template <bool BF16, bool GLU, bool SCATTER>
__device__ __forceinline__ void epilogue_row(const KParams &p, uint32_t tbase, bool valid,
                                             int64_t orow, float g, int n0, float *stage) {
    constexpr int OUT_COLS = GLU ? BN / 2 : BN;
    if constexpr (SCATTER && !GLU) {
        // The warp's 32 rows x 32 columns of each chunk go through shared memory (row stride
        // 33 floats: conflict-free both ways), so that each red.global.add.v4.f32 instruction
        // covers 4 rows x 128 contiguous bytes of out instead of 16 bytes in each of 32 rows.
        const int lane = threadIdx.x & 31;
        const int rsub = lane >> 3, cc = (lane & 7) * 4;
#pragma unroll 1
        for (int c = 0; c < OUT_COLS / 32; ++c) {
            uint32_t av[32];
            dev::tmem_ld32(tbase + c * 32, av);
            dev::tmem_ld_wait();
            const int col0 = n0 + c * 32;
#pragma unroll
            for (int j = 0; j < 32; ++j) stage[lane * 33 + j] = g * __uint_as_float(av[j]);
            __syncwarp();
#pragma unroll
            for (int pass = 0; pass < 8; ++pass) {
                const int rr = pass * 4 + rsub;
                const bool rv = __shfl_sync(0xffffffffu, valid, rr);
                const long long ro = __shfl_sync(0xffffffffu, (long long)orow, rr);
                if (rv && col0 + cc < p.N) {
                    const float *sv = stage + rr * 33 + cc;
                    dev::red_add_v4(reinterpret_cast<float *>(p.out) + ro * p.N + col0 + cc,
                                    sv[0], sv[1], sv[2], sv[3]);
                }
            }
            __syncwarp();
        }
        return;
    }
    if constexpr (GLU) {
#pragma unroll 1
        for (int c = 0; c < OUT_COLS / 32; ++c) {
            uint32_t gv[32], uv[32];
            dev::tmem_ld32(tbase + c * 32, gv);
            dev::tmem_ld32(tbase + OUT_COLS + c * 32, uv);
            dev::tmem_ld_wait();
            const int col0 = n0 + c * 32;
            if (valid && col0 < p.N) {
                float hv[32];
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    hv[j] = g * silu_f(__uint_as_float(gv[j])) * __uint_as_float(uv[j]);
                if (BF16) {
                    __nv_bfloat16 *dst =
                        reinterpret_cast<__nv_bfloat16 *>(p.out) + orow * p.N + col0;
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        if (col0 + v * 8 < p.N) {
                            uint4 pk;
                            uint32_t *pw = reinterpret_cast<uint32_t *>(&pk);
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                __nv_bfloat162 t2 = __floats2bfloat162_rn(
                                    hv[v * 8 + 2 * j], hv[v * 8 + 2 * j + 1]);
                                pw[j] = *reinterpret_cast<uint32_t *>(&t2);
                            }
                            *reinterpret_cast<uint4 *>(dst + v * 8) = pk;
                        }
                    }
                } else {
                    float *dst = reinterpret_cast<float *>(p.out) + orow * p.N + col0;
#pragma unroll
                    for (int v = 0; v < 8; ++v)
                        if (col0 + v * 4 < p.N)
                            *reinterpret_cast<float4 *>(dst + v * 4) = make_float4(
                                hv[v * 4], hv[v * 4 + 1], hv[v * 4 + 2], hv[v * 4 + 3]);
                }
            }
        }
    } else {
#pragma unroll 1
        for (int c = 0; c < OUT_COLS / 32; ++c) {
            uint32_t av[32];
            dev::tmem_ld32(tbase + c * 32, av);
            dev::tmem_ld_wait();
            const int col0 = n0 + c * 32;
            if (valid && col0 < p.N) {
                if (BF16) {
                    __nv_bfloat16 *dst =
                        reinterpret_cast<__nv_bfloat16 *>(p.out) + orow * p.N + col0;
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        if (col0 + v * 8 < p.N) {
                            uint4 pk;
                            uint32_t *pw = reinterpret_cast<uint32_t *>(&pk);
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                __nv_bfloat162 t2 = __floats2bfloat162_rn(
                                    g * __uint_as_float(av[v * 8 + 2 * j]),
                                    g * __uint_as_float(av[v * 8 + 2 * j + 1]));
                                pw[j] = *reinterpret_cast<uint32_t *>(&t2);
                            }
                            *reinterpret_cast<uint4 *>(dst + v * 8) = pk;
                        }
                    }
                } else {
                    float *dst = reinterpret_cast<float *>(p.out) + orow * p.N + col0;
#pragma unroll
                    for (int v = 0; v < 8; ++v)
                        if (col0 + v * 4 < p.N)
                            *reinterpret_cast<float4 *>(dst + v * 4) =
                                make_float4(g * __uint_as_float(av[v * 4]),
                                            g * __uint_as_float(av[v * 4 + 1]),
                                            g * __uint_as_float(av[v * 4 + 2]),
                                            g * __uint_as_float(av[v * 4 + 3]));
                }
            }
        }
    }
}

// SwiGLU backward in the epilogue of the fused gate+up GEMM (MLP backward): the accumulator holds
// a = x W_gate_e[e] in columns 0..127 and b = x W_up[e] in 128..255 for output columns n0.. of
// slot `slot` (route `route`, router weight g). With dh = g * dh_u (dh_u = the ungated gradient
// of h, read from bwd_dh) and h = silu(a) * b recomputed in fp32:
//   dw[route] += dh_u . h  (atomically: one partial per N tile)
//   da = dh * b * silu'(a), silu'(z) = sig(z) (1 + z (1 - sig(z)));  db = dh * silu(a)
// written as bf16 to out[out_row][n0 + c] and out[out_row][N + n0 + c] (row stride 2N).
__device__ __forceinline__ void glu_bwd_row(const KParams &p, uint32_t tbase, bool valid,
                                            int64_t slot, int64_t route, float g, int64_t out_row,
                                            int n0) {
    constexpr int HALF = BN / 2;
    float dw_acc = 0.f;
    const __nv_bfloat16 *dh_row = static_cast<const __nv_bfloat16 *>(p.bwd_dh) + slot * p.N;
    __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(p.out) + out_row * (2 * (int64_t)p.N);
#pragma unroll 1
    for (int c = 0; c < HALF / 32; ++c) {
        uint32_t av[32], bv[32];
        dev::tmem_ld32(tbase + c * 32, av);
        dev::tmem_ld32(tbase + HALF + c * 32, bv);
        dev::tmem_ld_wait();
        const int col0 = n0 + c * 32;
        if (!valid || col0 >= p.N) continue;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            if (col0 + v * 8 >= p.N) break;
            const uint4 u = *reinterpret_cast<const uint4 *>(dh_row + col0 + v * 8);
            const __nv_bfloat162 *hp = reinterpret_cast<const __nv_bfloat162 *>(&u);
            float da[8], db[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float2 d2 = __bfloat1622float2(hp[j >> 1]);
                const float du = (j & 1) ? d2.y : d2.x;
                const float a = __uint_as_float(av[v * 8 + j]);
                const float b = __uint_as_float(bv[v * 8 + j]);
                const float sg = 1.0f / (1.0f + __expf(-a));
                const float sl = a * sg;
                dw_acc = fmaf(du, sl * b, dw_acc);
                const float dh = g * du;
                da[j] = dh * b * sg * (1.0f + a * (1.0f - sg));
                db[j] = dh * sl;
            }
            uint4 pa, pb;
            uint32_t *wa = reinterpret_cast<uint32_t *>(&pa), *wb = reinterpret_cast<uint32_t *>(&pb);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                __nv_bfloat162 ta = __floats2bfloat162_rn(da[2 * j], da[2 * j + 1]);
                __nv_bfloat162 tb = __floats2bfloat162_rn(db[2 * j], db[2 * j + 1]);
                wa[j] = *reinterpret_cast<uint32_t *>(&ta);
                wb[j] = *reinterpret_cast<uint32_t *>(&tb);
            }
            *reinterpret_cast<uint4 *>(o + col0 + v * 8) = pa;
            *reinterpret_cast<uint4 *>(o + p.N + col0 + v * 8) = pb;
        }
    }
    if (valid) atomicAdd(p.bwd_dw + route, dw_acc);
}

}  // namespace gemm
}  // namespace moe
