// Attention core of Mixture of Attention (ScatterMoE guide, "2. Generalization to Mixture of
// Attention (MoA)"; the ScatterMoE abstract's MoA demonstration). The routed query projection
// leaves q in slot order, one row per (token, selected expert); keys and values are shared by all
// experts, one row per token. For route i (token s = i / k) with slot p = sparse_rows[i] and head h:
//   o[p, h] = sum_{t <= s} softmax_t(q[p, h] . K[t, h] / sqrt(dh)) V[t, h]
// i.e. causal attention in which every query row carries its own token position. The output stays
// in slot order for the routed output projection (grouped in, gated scatter-add out).
#include "moe_internal.cuh"

#include <cuda_bf16.h>
#include <math_constants.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <mutex>

namespace moe {
namespace {

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&v);
}

// =============================================================================================
// tcgen05 attention core
// =============================================================================================
// Query rows in route order: tile t holds routes [128 t, 128 t + 128), i.e. the k routes of 128/k
// consecutive tokens, so a tile's rows share nearly one causal limit and the cost of a tile grows
// with t. Row i reads q from slot sparse_rows[i] and writes o there. A work item is a pair of
// adjacent tiles (2u, 2u + 1) and one head; both tiles walk the key blocks the later tile needs
// (the earlier one's extra keys are masked). Items run in order of decreasing cost, dealt to
// persistent CTAs forwards in even rounds and backwards in odd rounds.
//
// Roles (320 threads):
//   warp 0     loads blocks of 128 keys of K and V by TMA (two stages each; K runs one block ahead
//              of V, since a K block is released by its score MMAs and a V block by its P V MMAs);
//   warp 1     issues the MMAs, alternating the tiles: for block j and tile x, O_x += P_x V (block
//              j - 1), then S_x = Q_x K^T (block j). Each tile has one TMEM score buffer; P is
//              written over it and read from TMEM as the A operand of P V, so the score MMA of
//              block j, issued after that P V, may overwrite it (tcgen05 MMAs of one thread run in
//              issue order). While one tile's softmax runs, the tensor cores work on the other's;
//   warps 2-5  the softmax group of tile 0, warps 6-9 that of tile 1: a thread owns one query row
//              (= its TMEM lane). It reads its 128 scores (two halves of 64 columns), masks keys past
//              its token, keeps a reference maximum that moves only when the row maximum exceeds
//              it by more than 2^8 (the exponentials stay below 256), writes the bf16
//              probabilities over the score buffer and rescales its O row when the reference
//              moved. After the last block it normalises O by the row sum and stores bf16 rows to
//              the slots; Q of its next tile is gathered by cp.async as soon as the tile's last
//              score MMA has completed.
namespace tc {

constexpr int BM = 128;                   // query rows per tile (two tiles per item)
constexpr int BN = 128;                   // keys per block
constexpr int THREADS = 320;              // producer warp, MMA warp, two softmax groups
constexpr int GROUP_WARPS = 4;
constexpr uint32_t CHUNK = 128u * 128u;   // 128 rows x 128 bytes, swizzled
constexpr uint32_t TMEM_COLS = 512;       // tile x: S / P at 128 x, O at 256 + 128 x
constexpr float kRescaleLog2 = 8.0f;
constexpr uint32_t NST = 2;               // stages of the K ring and of the V ring

template <int DH>
struct Layout {
    static constexpr int NCH = DH / 64;
    static constexpr uint32_t Q = NCH * CHUNK;   // one Q tile
    static constexpr uint32_t KV = NCH * CHUNK;  // one K (or V) block
    static constexpr uint32_t OFF_K = 2 * Q;
    static constexpr uint32_t OFF_V = OFF_K + NST * KV;
    static constexpr uint32_t OFF_BAR = OFF_V + NST * KV;
    static constexpr uint32_t SMEM = OFF_BAR + 256 + 1024;  // + barriers + alignment slack
    static constexpr uint32_t TX = KV;
};

struct Bars {
    uint64_t k_full[NST], k_empty[NST], v_full[NST], v_empty[NST];
    uint64_t s_full[2], p_full[2];  // [tile]: score block ready; P written (and O rescaled)
    uint64_t o_done[2];             // [tile]: the item's last P V completed
    uint64_t q_full[2], o_free[2];  // [tile]
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(Bars) <= 256, "barrier area");

struct Params {
    const __nv_bfloat16 *q;       // [R, HD] slot order
    const int32_t *sparse_rows;   // [R] route -> slot (negative: no slot)
    __nv_bfloat16 *o;             // [R, HD] slot order
    int64_t R, S, nitems;
    int32_t H, k, npairs;
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
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = dev::smem_u32(smem);
    Bars &bar = *reinterpret_cast<Bars *>(smem + L::OFF_BAR);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t HD = (int64_t)p.H * DH;

    if (threadIdx.x == 0) {
        for (uint32_t st = 0; st < NST; ++st) {
            dev::mbar_init(&bar.k_full[st], 1);
            dev::mbar_init(&bar.k_empty[st], 1);
            dev::mbar_init(&bar.v_full[st], 1);
            dev::mbar_init(&bar.v_empty[st], 1);
        }
        for (int x = 0; x < 2; ++x) {
            dev::mbar_init(&bar.s_full[x], 1);
            dev::mbar_init(&bar.p_full[x], GROUP_WARPS);
            dev::mbar_init(&bar.o_done[x], 1);
            dev::mbar_init(&bar.q_full[x], GROUP_WARPS);
            dev::mbar_init(&bar.o_free[x], GROUP_WARPS);
        }
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
    // round r of this CTA's items: items are in order of decreasing cost, dealt to the CTAs
    // forwards in even rounds and backwards in odd rounds
    auto item_of = [&](int r) {
        const int64_t G = gridDim.x;
        return (int64_t)r * G + ((r & 1) ? G - 1 - blockIdx.x : blockIdx.x);
    };
    // item -> (tile pair, head); blocks of 128 keys the pair needs (up to its last token)
    auto pair_of = [&](int64_t it) { return (int64_t)p.npairs - 1 - it / p.H; };
    auto head_of = [&](int64_t it) { return (int)(it % p.H); };
    auto nblocks = [&](int64_t pair) {
        const int64_t last = min(p.R, (2 * pair + 2) * BM) - 1;
        return (int)((last / p.k) / BN) + 1;
    };

    if (warp == 0) {
        // ---------------------------------------------------------------- K/V producer
        if (lane == 0) {
            // bit st: K stage st; bit NST + st: V stage st
            uint32_t issued = 0, last_par = 0;
            bool ok = true;
            auto load = [&](bool is_v, uint32_t gb, int h, int jb) {
                const uint32_t st = gb % NST;
                uint64_t *empty = is_v ? &bar.v_empty[st] : &bar.k_empty[st];
                uint64_t *full = is_v ? &bar.v_full[st] : &bar.k_full[st];
                if (gb >= NST && !dev::mbar_wait(empty, ((gb - NST) / NST) & 1u, abort, p.status,
                                                 p.wait_limit_ns, kKernelAttention))
                    return false;
                dev::mbar_arrive_expect_tx(full, L::TX);
                uint8_t *dst = smem + (is_v ? L::OFF_V : L::OFF_K) + st * L::KV;
#pragma unroll
                for (int c = 0; c < L::NCH; ++c)
                    dev::tma_load_2d(dst + c * CHUNK, &tmKV, full,
                                     (int32_t)((is_v ? HD : 0) + h * DH + c * 64),
                                     (int32_t)(jb * BN));
                const uint32_t bit = (is_v ? NST : 0u) + st;
                issued |= 1u << bit;
                last_par = (last_par & ~(1u << bit)) | (((gb / NST) & 1u) << bit);
                return true;
            };
            uint32_t g = 0, vg = 0;
            int vh = -1, vj = 0;  // the block whose V is still to be loaded
            for (int r = 0; item_of(r) < p.nitems && ok; ++r) {
                const int64_t it = item_of(r);
                const int h = head_of(it);
                const int n = nblocks(pair_of(it));
                for (int j = 0; j < n; ++j, ++g) {
                    if (!load(false, g, h, j) || (vh >= 0 && !load(true, vg, vh, vj))) {
                        ok = false;
                        break;
                    }
                    vh = h;
                    vj = j;
                    vg = g;
                }
            }
            if (ok && vh >= 0) load(true, vg, vh, vj);
            // teardown: every load issued must land before the CTA may exit
            for (uint32_t bit = 0; bit < 2 * NST; ++bit)
                if (issued & (1u << bit))
                    dev::mbar_wait(bit < NST ? &bar.k_full[bit] : &bar.v_full[bit - NST],
                                   (last_par >> bit) & 1u, nullptr, p.status, kDrainLimitNs,
                                   kKernelAttention);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            auto wait = [&](uint64_t *b, uint32_t par) {
                return dev::mbar_wait(b, par, abort, p.status, p.wait_limit_ns, kKernelAttention);
            };
            // O_x += P_x V for global block gp (the first block of an item overwrites O_x, after
            // the softmax group has read the previous item's O_x)
            auto pv = [&](int x, uint32_t gp, bool first, uint32_t icnt) {
                const uint32_t vs = gp % NST;
                if ((x == 0 && !wait(&bar.v_full[vs], (gp / NST) & 1u)) ||
                    !wait(&bar.p_full[x], gp & 1u) ||
                    (first && icnt > 0 && !wait(&bar.o_free[x], (icnt - 1) & 1u)))
                    return false;
                dev::tc_fence_after();
                const uint32_t sV = sbase + L::OFF_V + vs * L::KV;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk)
                    dev::mma_bf16_ts(tmem + 256 + 128 * x, tmem + 128 * x + kk * 8,
                                     dev::sdesc(sV + kk * 2048, CHUNK, 1024, dev::kLayoutSw128),
                                     IDESC_O, (!first || kk > 0) ? 1u : 0u);
                return true;
            };
            auto score = [&](int x, uint32_t ks) {
                const uint32_t sQ = sbase + (uint32_t)x * L::Q;
                const uint32_t sK = sbase + L::OFF_K + ks * L::KV;
#pragma unroll
                for (int kk = 0; kk < DH / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * CHUNK + (kk & 3) * 32;
                    dev::mma_bf16(tmem + 128 * x,
                                  dev::sdesc(sQ + off, 16, 1024, dev::kLayoutSw128),
                                  dev::sdesc(sK + off, 16, 1024, dev::kLayoutSw128), IDESC_S,
                                  kk > 0 ? 1u : 0u);
                }
                dev::mma_commit(&bar.s_full[x]);
            };
            uint32_t g = 0, icnt = 0;
            bool ok = true;
            for (int r = 0; item_of(r) < p.nitems && ok; ++r, ++icnt) {
                const int n = nblocks(pair_of(item_of(r)));
                for (int j = 0; j < n && ok; ++j) {
                    const uint32_t gj = g + j, ks = gj % NST;
                    if (!wait(&bar.k_full[ks], (gj / NST) & 1u)) {
                        ok = false;
                        break;
                    }
                    for (int x = 0; x < 2; ++x) {
                        if (j >= 1 && !pv(x, gj - 1, j == 1, icnt)) {
                            ok = false;
                            break;
                        }
                        if (j == 0 && !wait(&bar.q_full[x], icnt & 1u)) {
                            ok = false;
                            break;
                        }
                        dev::tc_fence_after();
                        score(x, ks);
                    }
                    if (!ok) break;
                    dev::mma_commit(&bar.k_empty[ks]);
                    if (j >= 1) dev::mma_commit(&bar.v_empty[(gj - 1) % NST]);
                }
                if (!ok) break;
                const uint32_t gl = g + n - 1;
                for (int x = 0; x < 2 && ok; ++x) {
                    if (!pv(x, gl, n == 1, icnt)) {
                        ok = false;
                        break;
                    }
                    dev::mma_commit(&bar.o_done[x]);
                }
                if (!ok) break;
                dev::mma_commit(&bar.v_empty[gl % NST]);
                g += n;
            }
            // teardown: all issued MMAs complete before TMEM is released
            dev::mma_commit(&bar.drain);
            dev::mbar_wait(&bar.drain, 0, nullptr, p.status, kDrainLimitNs, kKernelAttention);
            dev::tc_fence_before();
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- softmax groups
        const int x = (warp - 2) >> 2;           // tile of the pair this group owns
        const int qw = warp & 3;                 // TMEM lane quarter this warp may access
        const int row = qw * 32 + lane;          // query row of the tile = TMEM lane
        const uint32_t tl = tmem + ((uint32_t)(qw * 32) << 16);
        const uint32_t s_col = 128 * x, o_col = 256 + 128 * x;
        const uint32_t sQ = sbase + (uint32_t)x * L::Q;
        auto wait = [&](uint64_t *b, uint32_t par) {  // warp-uniform bounded wait
            bool w = true;
            if (lane == 0)
                w = dev::mbar_wait(b, par, abort, p.status, p.wait_limit_ns, kKernelAttention);
            return __shfl_sync(0xffffffffu, w, 0) != 0;
        };
        // one arrival per warp, after every lane's preceding accesses (fenced by the caller)
        auto arrive = [&](uint64_t *b) {
            __syncwarp();
            if (lane == 0) dev::mbar_arrive(b);
        };
        auto slot_of = [&](int64_t pair) {
            const int64_t i = (2 * pair + x) * BM + row;
            const int32_t sl = i < p.R ? __ldg(p.sparse_rows + i) : -1;
            // -1 marks a route without a slot (its expert id was out of range); debug builds flag
            // any other slot outside [0, R)
            if (sl != -1 && !dev::debug_in_range(sl, p.R, p.status)) return (int64_t)-1;
            return (sl >= 0 && sl < p.R) ? (int64_t)sl : (int64_t)-1;
        };
        // this thread's row of Q for (pair, head) -> this group's Q tile (zeros without a slot)
        auto load_q = [&](int64_t pair, int h) {
            const int64_t sl = slot_of(pair);
            const __nv_bfloat16 *src = sl >= 0 ? p.q + sl * HD + (int64_t)h * DH : p.q;
#pragma unroll
            for (int u = 0; u < DH / 8; ++u)
                dev::cp_async16(sQ + sw_off(row, u), sl >= 0 ? src + u * 8 : p.q,
                                sl >= 0 ? 16u : 0u);
        };
        // the block's 128 scores -> registers (one wait for the four loads), keys past `pos`
        // set to -inf
        auto load_scores = [&](int key0, int pos, uint32_t (&sr)[BN / 32][32]) {
#pragma unroll
            for (int c = 0; c < BN / 32; ++c) dev::tmem_ld32(tl + s_col + 32 * c, sr[c]);
            dev::tmem_ld_wait();
            if (key0 + BN - 1 > pos) {
#pragma unroll
                for (int c = 0; c < BN; ++c)
                    if (key0 + c > pos) sr[c / 32][c % 32] = __float_as_uint(-CUDART_INF_F);
            }
        };
        uint32_t g = 0, icnt = 0;
        bool ok = true;
        int64_t it = item_of(0);
        if (it < p.nitems) {
            load_q(pair_of(it), head_of(it));
            dev::cp_async_wait_all();
            dev::fence_proxy_async_smem();
            arrive(&bar.q_full[x]);
        }
        for (int r = 0; it < p.nitems && ok; it = item_of(++r), ++icnt) {
            const int64_t pair = pair_of(it);
            const int h = head_of(it);
            const int n = nblocks(pair);
            const int64_t slot = slot_of(pair);
            const int pos = slot >= 0 ? (int)(((2 * pair + x) * BM + row) / p.k) : -1;
            const int64_t nit = item_of(r + 1);
            const bool has_next = nit < p.nitems;
            float m_ref = -CUDART_INF_F, l = 0.f;
            for (int j = 0; j < n && ok; ++j) {
                const uint32_t gj = g + j;
                if (!wait(&bar.s_full[x], gj & 1u)) {
                    ok = false;
                    break;
                }
                dev::tc_fence_after();
                // the tile's last score MMA has completed: its Q may be replaced
                if (j == n - 1 && has_next) load_q(pair_of(nit), head_of(nit));
                const int key0 = j * BN;
                uint32_t sr[BN / 32][32];
                load_scores(key0, pos, sr);
                // the row maximum over the block (8 independent chains)
                float pm[8];
#pragma unroll
                for (int t = 0; t < 8; ++t) pm[t] = __uint_as_float(sr[0][t]);
#pragma unroll
                for (int c = 8; c < BN; ++c)
                    pm[c % 8] = fmaxf(pm[c % 8], __uint_as_float(sr[c / 32][c % 32]));
                const float mx = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                                       fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
                const float mxs = mx * p.scale_log2;
                const bool need = mxs > m_ref + kRescaleLog2;
                float alpha = 1.f;
                if (need) {
                    alpha = ex2(m_ref - mxs);
                    m_ref = mxs;
                }
                const float mneg = m_ref == -CUDART_INF_F ? 0.f : -m_ref;
                // probabilities, written as bf16 pairs over the first 64 columns of the score
                // buffer (all scores are in registers by now)
                float ps[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    uint32_t pk[32];
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const int k0 = 64 * hh + 2 * c;
                        const float e0 = ex2(fmaf(__uint_as_float(sr[k0 / 32][k0 % 32]),
                                                  p.scale_log2, mneg));
                        const float e1 = ex2(fmaf(__uint_as_float(sr[(k0 + 1) / 32][(k0 + 1) % 32]),
                                                  p.scale_log2, mneg));
                        ps[(2 * c) % 8] += e0;
                        ps[(2 * c + 1) % 8] += e1;
                        pk[c] = pack_bf16(e0, e1);
                    }
                    dev::tmem_st32(tl + s_col + 32 * hh, pk);
                }
                const float sum = ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
                l = l * alpha + sum;
                // O holds P V of blocks < gj (complete: this block's score MMA was issued after
                // the previous P V): rescale the rows whose reference moved
                if (j >= 1 && __any_sync(0xffffffffu, need)) {
#pragma unroll
                    for (int c = 0; c < DH / 32; ++c) {
                        uint32_t o[32];
                        dev::tmem_ld32(tl + o_col + c * 32, o);
                        dev::tmem_ld_wait();
#pragma unroll
                        for (int t = 0; t < 32; ++t) o[t] = __float_as_uint(__uint_as_float(o[t]) * alpha);
                        dev::tmem_st32(tl + o_col + c * 32, o);
                    }
                }
                dev::tmem_st_wait();
                dev::tc_fence_before();
                arrive(&bar.p_full[x]);
            }
            if (!ok) break;
            // O complete after the item's last P V: normalise and store the row
            if (!wait(&bar.o_done[x], icnt & 1u)) break;
            dev::tc_fence_after();
            const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
            for (int c = 0; c < DH / 32; ++c) {
                uint32_t o[32];
                dev::tmem_ld32(tl + o_col + c * 32, o);
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
            arrive(&bar.o_free[x]);
            if (has_next) {
                dev::cp_async_wait_all();
                dev::fence_proxy_async_smem();
                arrive(&bar.q_full[x]);
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
    const uint32_t box[2] = {64, (uint32_t)tc::BN};  // 64 head columns x one key block
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
    const int64_t ntiles = (R + tc::BM - 1) / tc::BM;
    p.npairs = (int32_t)((ntiles + 1) / 2);
    p.nitems = (int64_t)p.npairs * H;
    p.scale_log2 = (float)(1.4426950408889634 / sqrt((double)DH));
    p.status = status;
    p.wait_limit_ns = kWaitLimitNs;
    const int grid = (int)std::min<int64_t>(num_sms(), p.nitems);
    kern<<<grid, tc::THREADS, L::SMEM, s>>>(m, p);
    return MOE_OK;
}

}  // namespace

int launch_moa_attention(const void *q, const void *kv, const int32_t *sparse_rows, void *o,
                         int64_t R, int64_t S, int32_t H, int32_t dh, int32_t k, unsigned *status,
                         cudaStream_t s) {
    if (R == 0) return MOE_OK;
    if (dh != 64 && dh != 128)
        return set_error(MOE_ERR_UNSUPPORTED, "moa attention: head size %d (64 or 128 are built)", dh);
    if (R >= (int64_t(1) << 31) - 2 * tc::BM || S >= (int64_t(1) << 31) - tc::BN)
        return set_error(MOE_ERR_INVALID_ARG, "moa attention: sizes too large");
    return dh == 128 ? launch_tc<128>(q, kv, sparse_rows, o, R, S, H, k, status, s)
                     : launch_tc<64>(q, kv, sparse_rows, o, R, S, H, k, status, s);
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
