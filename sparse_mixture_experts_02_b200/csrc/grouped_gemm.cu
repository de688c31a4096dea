// Scattered grouped GEMM on the sm_100a tensor cores (tcgen05 + TMEM + TMA), one kernel for
// every form of ParallelLinear(X, W, I, G) the library needs:
//
//   GEMM1 of the MoE MLP:   gathered x rows, W_gate_e and W_up side by side in one MMA (N = 256:
//                           128 gate columns + the same 128 up columns), SwiGLU in registers,
//                           h rows stored in slot (expert-grouped) order;
//   GEMM2 of the MoE MLP:   contiguous h rows, W_down, router-weight scaling, fp32 vector
//                           atomic scatter-add into token order;
//   moe_scatter_linear:     any of gather / contiguous input x scatter / grouped output.
//
// Sources: ScatterMoE guide ("ScatterMoE Guide: Fast Fused Kernels for Sparse MoE LLMs"),
// "The ParallelLinear Core Abstraction" figure (Step 1 indexed gather, Step 2 tile GEMM against
// W[expert], Step 3 gate scaling and scatter-add), "2. Grouped Coordinate Indexing Without
// Padding" (ceil(N_e / B_M) tiles per expert, the last one masked, no padding in memory) and
// "3. Assembling the ScatterMoE FFN Block" (SwiGLU, gate half first); the fused gate+up
// mainloop follows the abstract of "Cross-Platform Fused MoE Dispatch in Triton"; the per-tile
// expert id follows "Inside the Flash-MoE Kernel: Fused Tile-Level Dispatch".
//
// Design (B200): persistent, one CTA per SM, 6 warps:
//   warp 0      TMA producer: B tiles by 3-D tensor map (N, K, expert); contiguous A tiles
//               (slot-ordered rows) by a 2-D box.
//   warps 6-9   (gathered A only) row gatherers: 128 threads copy the stage's 128 token rows
//               (row = x[sorted_rows[p] / k]) with 16-byte cp.async straight into the 128-byte
//               swizzled layout, so no [S*k, D] copy of x ever exists. (TMA tile::gather4 was
//               measured at ~7x the cost per row of a box load here, leaving the tensor pipe
//               80% idle; the LSU path keeps the gather off the TMA unit.)
//   warp 1      TMEM owner (512 columns = two 128 x 256 fp32 accumulators) and MMA issuer
//               (one thread): 4 x tcgen05.mma (M=128, N=256, K=32 bytes) per 128-byte K stage.
//   warps 2-5   epilogue: tcgen05.ld of the accumulator (thread = tile row), then SwiGLU + bf16
//               store, or gate * acc and red.global.add.v4.f32 into out[token].
// Stages: 4 x (A 16 KB + B 32 KB), 128-byte swizzle; A is K-major, B (weights, N contiguous)
// is MN-major, or K-major for the transposed weights of the backward pass (BKM: a weight
// [E, Din, Dout] read as W^T, one 64 x 256 box per stage). Two accumulators let the epilogue of
// tile i overlap the mainloop of tile i+1.
// Tile schedule: every CTA derives it from expert_offsets on the device (no host sync):
// tiles are ordered expert-major, then N tile, then M tile, so the CTAs running at one time
// share expert weight tiles and gathered rows through L2. Waits are bounded (see mbar_wait).
#include "gemm_common.cuh"

#include <stdio.h>
#include <mutex>

namespace moe {
namespace {

using namespace gemm;

// Router epilogue of one token row (the calling thread's TMEM lane): the K largest of
// logit + bias over the E columns, in descending order with ties to the smaller expert id, and
// the softmax over those K logits.
// Each logit becomes one 64-bit key: the logit's bits in an order-preserving unsigned form above
// the complement of the expert id. Keys then compare exactly like (logit descending, id
// ascending) and no two are equal, so the top K is a branch-free insertion: every step keeps the
// larger of a list entry and the carried key and carries the smaller on. NaN counts as -inf and
// -0 as +0, as in a floating-point comparison. (A per-expert insertion that compared logits and
// ids in branches took 23-44 us per 128-token tile, most of the router's time.)
template <int K>
__device__ __forceinline__ void router_row(const KParams &p, uint32_t tbase, int E, int64_t srow,
                                           bool valid) {
    uint64_t top[K];
#pragma unroll
    for (int q = 0; q < K; ++q) top[q] = 0;  // below every key (-inf maps above 0)
    for (int c = 0; c * 32 < E; ++c) {
        uint32_t av[32];
        dev::tmem_ld32(tbase + c * 32, av);
        dev::tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int e = c * 32 + j;
            if (e < E) {
                float v = __uint_as_float(av[j]);
                if (p.bias != nullptr) v += __ldg(p.bias + e);
                if (isnan(v)) v = -INFINITY;
                if (v == 0.0f) v = 0.0f;
                const uint32_t u = __float_as_uint(v);
                const uint32_t o = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
                uint64_t key = ((uint64_t)o << 32) | (uint64_t)(~(uint32_t)e);
#pragma unroll
                for (int q = 0; q < K; ++q) {
                    const bool up = key > top[q];
                    const uint64_t hi = up ? key : top[q];
                    key = up ? top[q] : key;
                    top[q] = hi;
                }
            }
        }
    }
    if (!valid) return;
    float tv[K];
#pragma unroll
    for (int q = 0; q < K; ++q) {
        const uint32_t o = (uint32_t)(top[q] >> 32);
        tv[q] = __uint_as_float((o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o);
    }
    const float m = tv[0];
    float den = 0.f;
#pragma unroll
    for (int q = 0; q < K; ++q) den += expf(tv[q] - m);
#pragma unroll
    for (int q = 0; q < K; ++q) {
        p.top_e[srow * K + q] = (int32_t)(~(uint32_t)top[q]);
        p.top_w[srow * K + q] = expf(tv[q] - m) / den;
    }
}

template <bool BF16, bool GATHER, bool GLU, bool SCATTER, bool ROUTER, bool BKM, bool GBWD>
__global__ void __launch_bounds__(GATHER ? THREADS + GATHER_THREADS : THREADS, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                    const __grid_constant__ CUtensorMap tmB0,
                    const __grid_constant__ CUtensorMap tmB1, const KParams p) {
    constexpr int EB = BF16 ? 2 : 4;          // input element bytes
    constexpr int BK = KBYTES / EB;           // K elements per stage
    constexpr int CW = KBYTES / EB;           // N elements per 128-byte B chunk
    constexpr int NCH = BN / CW;              // B chunks per stage
    constexpr int CHUNK = BK * KBYTES;        // bytes of one B chunk
    constexpr int B_KSTEP = (32 / EB) * KBYTES;  // bytes of B per MMA K step (32 bytes of K)
    constexpr int OUT_COLS = GLU ? BN / 2 : BN;  // output columns per tile
    static_assert(!(BKM && (GLU || ROUTER)), "K-major B is for the plain grouped GEMM");
    static_assert(!GBWD || (BF16 && GLU && !SCATTER && !ROUTER), "GLU backward epilogue form");
    constexpr uint32_t IDESC = dev::idesc_f32acc(BF16, BM, BN, !BKM);
    // A tile with at most 64 rows (an expert's short last tile) runs an M=64 MMA: half the tensor
    // work; its accumulator rows 16j + i (i < 16) sit in TMEM lanes 32j + i.
    constexpr uint32_t IDESC64 = dev::idesc_f32acc(BF16, 64, BN, !BKM);
    // B (weights, N contiguous) is MN-major: 128-byte swizzle for bf16 (8-row atoms of 1024 B);
    // tf32 needs the 32-byte-unit variant (4-row atoms of 512 B).
    constexpr uint32_t B_LAYOUT = BF16 ? dev::kLayoutSw128 : dev::kLayoutSw128Base32;
    constexpr uint32_t B_SBO = BF16 ? 1024 : 512;
    static_assert(NCH * CHUNK == B_BYTES, "B stage size");

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    SmemTail &st = *reinterpret_cast<SmemTail *>(smem + STAGE_AREA);
    // the router's B is only ceil(E/64) chunks: it runs more, smaller stages in the same space
    const int nst = ROUTER ? p.stages : STAGES;
    const size_t sbytes = ROUTER ? (size_t)p.stage_bytes : (size_t)STAGE_BYTES;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = p.E;
    // the router is the forward's first kernel: it clears the status word
    if (ROUTER && blockIdx.x == 0 && threadIdx.x == 0 && p.status != nullptr) *p.status = 0u;

    if (threadIdx.x == 0) {
        for (int s = 0; s < nst; ++s) {
            // full: the TMA thread's expect_tx arrival (+ one cp.async arrival per gatherer)
            dev::mbar_init(&st.full[s], GATHER ? 1 + GATHER_THREADS : 1);
            dev::mbar_init(&st.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            dev::mbar_init(&st.tfull[b], 1);
            dev::mbar_init(&st.tempty[b], 4);
        }
        dev::mbar_init(&st.drain, 1);
        st.abort = 0;
        dev::fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        dev::prefetch_tmap(&tmA);
        dev::prefetch_tmap(&tmB0);
        if (GLU || BKM) dev::prefetch_tmap(&tmB1);
    }
    if (warp == 1) {
        dev::tmem_alloc(&st.tmem_base, TMEM_COLS);
        dev::tmem_relinquish();
        dev::tc_fence_before();
    }
    if constexpr (ROUTER) {
        // one "expert" holding all S rows: tiles are the 128-token blocks of x
        if (threadIdx.x == 0) {
            st.off[0] = 0;
            st.off[1] = (int32_t)p.S;
            st.tstart[0] = 0;
            st.tstart[1] = (int32_t)((p.S + BM - 1) / BM);
        }
        __syncthreads();
    } else {
        for (int e = threadIdx.x; e <= E; e += blockDim.x) st.off[e] = __ldg(p.offsets + e);
        __syncthreads();
        if (threadIdx.x == 0) {
            build_schedule<BM>(st.off, st.tstart, E, p.n_tiles);
            debug_check_offsets(st.off, st.tstart, E, p.R, p.status);
        }
        __syncthreads();
    }
    dev::tc_fence_after();
    const uint32_t tmem_base = st.tmem_base;
    const int E_sched = ROUTER ? 1 : E;
    const int total = st.tstart[E_sched];
    const int nch = ROUTER ? p.b_chunks : NCH;
    const uint32_t stage_tx = (uint32_t)((GATHER ? 0 : A_BYTES) + nch * CHUNK);
    const uint32_t idesc = ROUTER ? dev::idesc_f32acc(BF16, BM, (uint32_t)(nch * CW), true) : IDESC;
    volatile int *abort = &st.abort;

    if (warp == 0) {
        // ------------------------------------------------------------------ TMA producer
        uint32_t s = 0, ph = 0;
        uint32_t issued = 0, last_par = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
            const TileInfo ti = decode_tile<BM>(t, st.off, st.tstart, E_sched);
            const int n0 = ti.n_idx * OUT_COLS;
            for (int kb = 0; kb < p.num_kb; ++kb) {
                bool w = true;
                if (lane == 0)
                    w = dev::mbar_wait(&st.empty[s], ph ^ 1u, abort, p.status, p.wait_limit_ns,
                                       kKernelGemm);
                w = __shfl_sync(0xffffffffu, w, 0);
                if (!w) {
                    ok = false;
                    break;
                }
                uint8_t *sA = smem + (size_t)s * sbytes;
                uint8_t *sB = sA + A_BYTES;
                if (lane == 0) dev::mbar_arrive_expect_tx(&st.full[s], stage_tx);
                __syncwarp();
                const int kc = kb * BK;
                if (!GATHER && lane == 0)
                    dev::tma_load_2d(sA, &tmA, &st.full[s], kc,
                                     ti.row_begin + p.a_row_pad * ti.e);
                if (BKM && lane == 0) {
                    const bool hi = kc >= p.k_split;
                    dev::tma_load_3d(sB, hi ? &tmB1 : &tmB0, &st.full[s], hi ? kc - p.k_split : kc,
                                     n0, ti.e);
                } else if (lane == 0) {
#pragma unroll
                    for (int c = 0; c < NCH; ++c) {
                        if (c >= nch) break;
                        if (GLU) {
                            const int half = NCH / 2;
                            const CUtensorMap *m = c < half ? &tmB0 : &tmB1;
                            dev::tma_load_3d(sB + c * CHUNK, m, &st.full[s],
                                             n0 + (c % half) * CW, kc, ti.e);
                        } else {
                            dev::tma_load_3d(sB + c * CHUNK, &tmB0, &st.full[s], n0 + c * CW, kc,
                                             ti.e);
                        }
                    }
                }
                issued |= 1u << s;
                last_par = (last_par & ~(1u << s)) | (ph << s);
                if (++s == (uint32_t)nst) {
                    s = 0;
                    ph ^= 1u;
                }
            }
        }
        // teardown: every load this warp issued must land before the CTA may exit
        if (lane == 0) {
            for (int s2 = 0; s2 < nst; ++s2)
                if (issued & (1u << s2))
                    dev::mbar_wait(&st.full[s2], (last_par >> s2) & 1u, nullptr, p.status,
                                   kDrainLimitNs, kKernelGemm);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            uint32_t s = 0, ph = 0;
            int it = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++it) {
                const uint32_t b = it & 1, aph = (it >> 1) & 1;
                if (!dev::mbar_wait(&st.tempty[b], aph ^ 1u, abort, p.status, p.wait_limit_ns,
                                    kKernelGemm))
                    break;
                dev::tc_fence_after();
                const uint32_t d_tmem = tmem_base + b * BN;
                uint32_t tile_idesc = idesc;
                if (!ROUTER && decode_tile<BM>(t, st.off, st.tstart, E_sched).rows <= 64)
                    tile_idesc = IDESC64;
                for (int kb = 0; kb < p.num_kb; ++kb) {
                    if (!dev::mbar_wait(&st.full[s], ph, abort, p.status, p.wait_limit_ns,
                                        kKernelGemm)) {
                        ok = false;
                        break;
                    }
                    dev::tc_fence_after();
                    if (GATHER) dev::fence_proxy_async_smem();  // cp.async rows -> tensor core
                    const uint32_t sA = dev::smem_u32(smem + (size_t)s * sbytes);
                    const uint32_t sB = sA + A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < KBYTES / 32; ++kk) {
                        const uint64_t ad =
                            dev::sdesc(sA + kk * 32, 16, 1024, dev::kLayoutSw128);
                        const uint64_t bd =
                            BKM ? dev::sdesc(sB + kk * 32, 16, 1024, dev::kLayoutSw128)
                                : dev::sdesc(sB + kk * B_KSTEP, CHUNK, B_SBO, B_LAYOUT);
                        if (BF16) dev::mma_bf16(d_tmem, ad, bd, tile_idesc, (kb | kk) != 0);
                        else dev::mma_tf32(d_tmem, ad, bd, tile_idesc, (kb | kk) != 0);
                    }
                    dev::mma_commit(&st.empty[s]);
                    if (++s == (uint32_t)nst) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                dev::mma_commit(&st.tfull[b]);
            }
            // teardown: all issued MMAs complete before TMEM is released
            dev::mma_commit(&st.drain);
            dev::mbar_wait(&st.drain, 0, nullptr, p.status, kDrainLimitNs, kKernelGemm);
            dev::tc_fence_before();
        }
        __syncwarp();
    } else if (GATHER && warp >= THREADS / 32) {
        // ------------------------------------------------------------------ row gatherers
        // thread -> 8 rows of the 128-row stage (rows gw*32 + 4i + lane/8) and one 16-byte chunk
        // (lane % 8) of each row's 128 bytes, so a warp instruction covers 4 whole rows.
        const int gw = warp - THREADS / 32;
        const int chunk = lane & 7;
        const int rsub = lane >> 3;
        const int64_t row_bytes = (int64_t)p.K * EB;
        const uint8_t *xa = reinterpret_cast<const uint8_t *>(p.A);
        // sorted_rows entries of this thread's 8 rows of tile t (tail rows repeat a valid row)
        auto fetch_rows = [&](int t, int *ent) {
            const TileInfo ti = decode_tile<BM>(t, st.off, st.tstart, E_sched);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int r = gw * 32 + i * 4 + rsub;
                ent[i] = __ldg(p.sorted_rows + ti.row_begin + min(r, ti.rows - 1));
            }
        };
        // x row pointers of tile t from its entries; returns the tile's rows
        auto row_ptrs = [&](int t, const int *ent, const uint8_t **src) {
            const TileInfo ti = decode_tile<BM>(t, st.off, st.tstart, E_sched);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                // debug builds: a route outside [0, S*k) reads row 0 instead (and is flagged)
                const int en = dev::debug_in_range(ent[i], (int64_t)p.S * p.k, p.status) ? ent[i] : 0;
                src[i] = xa + (int64_t)(en / p.k) * row_bytes;
            }
            return ti.rows;
        };
        // Shared memory is saturated by the tensor core, so a tile's schedule lookups, index
        // loads and divisions take ~2 us: the next tile's pointers are formed after the current
        // tile's second stage is issued, and its entries are loaded a tile earlier still, so
        // nothing but a register swap sits between two tiles' copies.
        const int t0 = blockIdx.x, tstep = gridDim.x;
        int ent[8];
        const uint8_t *src[8], *nsrc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) src[i] = nsrc[i] = xa;
        int rows = 0, nrows = 0;
        if (t0 < total) {
            fetch_rows(t0, ent);
            rows = row_ptrs(t0, ent, src);
            if (t0 + tstep < total) fetch_rows(t0 + tstep, ent);
        }
        const int prep_kb = min(1, p.num_kb - 1);
        uint32_t s = 0, ph = 0;
        bool ok = true;
        for (int t = t0; t < total && ok; t += tstep) {
            for (int kb = 0; kb < p.num_kb; ++kb) {
                bool w = true;
                if (lane == 0)
                    w = dev::mbar_wait(&st.empty[s], ph ^ 1u, abort, p.status, p.wait_limit_ns,
                                       kKernelGemm);
                w = __shfl_sync(0xffffffffu, w, 0);
                if (!w) {
                    ok = false;
                    break;
                }
                const uint32_t sA = dev::smem_u32(smem + (size_t)s * sbytes);
                const int64_t cb = (int64_t)kb * KBYTES + chunk * 16;
                const uint32_t nbytes = cb < row_bytes ? 16u : 0u;  // zero-fill past K
                // rows past the tile's end are not copied: an A row only feeds its own output
                // row, which the epilogue discards (an M=64 tile's MMA reads rows 0-63 only)
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = gw * 32 + i * 4 + rsub;
                    const uint32_t dst = sA + r * KBYTES + ((chunk ^ (r & 7)) << 4);
                    if (r < rows) dev::cp_async16(dst, nbytes ? src[i] + cb : src[i], nbytes);
                }
                dev::cp_async_arrive_noinc(&st.full[s]);
                if (kb == prep_kb && t + tstep < total) {
                    nrows = row_ptrs(t + tstep, ent, nsrc);
                    if (t + 2 * tstep < total) fetch_rows(t + 2 * tstep, ent);
                }
                if (++s == (uint32_t)nst) {
                    s = 0;
                    ph ^= 1u;
                }
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) src[i] = nsrc[i];
            rows = nrows;
        }
        dev::cp_async_wait_all();
    } else {
        // ------------------------------------------------------------------ epilogue
        zero_side_job(p, threadIdx.x - 64, 128);
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        const int r_full = q * 32 + lane;
        const int r_half = lane < 16 ? q * 16 + lane : BM;  // M=64 layout; BM = no row
        int it = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x, ++it) {
            const TileInfo ti = decode_tile<BM>(t, st.off, st.tstart, E_sched);
            const uint32_t b = it & 1, aph = (it >> 1) & 1;
            bool w = true;
            if (lane == 0)
                w = dev::mbar_wait(&st.tfull[b], aph, abort, p.status, p.wait_limit_ns,
                                   kKernelGemm);
            w = __shfl_sync(0xffffffffu, w, 0);
            if (!w) break;
            dev::tc_fence_after();
            const int r = (!ROUTER && ti.rows <= 64) ? r_half : r_full;
            const int prow = ti.row_begin + r;
            bool valid = r < ti.rows && prow >= 0 && prow < p.R;
            int64_t orow = prow;
            float g = 1.0f;
            if (valid && (SCATTER || p.gates != nullptr)) {
                const int i = __ldg(p.sorted_rows + prow);
                if (SCATTER) orow = i / p.k;
                if (p.gates != nullptr && i >= 0 && i < p.R) g = __ldg(p.gates + i);
                // a slot whose route is outside [0, R) is skipped rather than written anywhere
                if (!dev::debug_in_range(i, p.R, p.status) || i < 0 || i >= p.R) valid = false;
            }
            const int n0 = ti.n_idx * OUT_COLS;
            const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + b * BN;
            if constexpr (ROUTER) {
                switch (p.k) {
                    case 1: router_row<1>(p, tbase, E, ti.row_begin + r, r < ti.rows); break;
                    case 2: router_row<2>(p, tbase, E, ti.row_begin + r, r < ti.rows); break;
                    case 3: router_row<3>(p, tbase, E, ti.row_begin + r, r < ti.rows); break;
                    case 4: router_row<4>(p, tbase, E, ti.row_begin + r, r < ti.rows); break;
                    case 5: router_row<5>(p, tbase, E, ti.row_begin + r, r < ti.rows); break;
                    case 6: router_row<6>(p, tbase, E, ti.row_begin + r, r < ti.rows); break;
                    case 7: router_row<7>(p, tbase, E, ti.row_begin + r, r < ti.rows); break;
                    default: router_row<8>(p, tbase, E, ti.row_begin + r, r < ti.rows); break;
                }
            } else if constexpr (GBWD) {
                const int64_t route = valid ? (int64_t)__ldg(p.sorted_rows + prow) : 0;
                glu_bwd_row(p, tbase, valid, prow, route, g,
                            prow + (int64_t)p.out_row_pad * ti.e, n0);
            } else {
                epilogue_row<BF16, GLU, SCATTER>(p, tbase, valid, orow, g, n0, st.stage[q]);
            }
            dev::tc_fence_before();
            __syncwarp();
            if (lane == 0) dev::mbar_arrive(&st.tempty[b]);
        }
    }

    __syncthreads();
    if (warp == 1) {
        dev::tc_fence_after();
        dev::tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

__global__ void debug_wait_kernel(int64_t limit_ns, unsigned *status) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        dev::mbar_init(&bar, 1);  // nothing ever arrives
        abort_flag = 0;
        dev::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0)
        dev::mbar_wait(&bar, 0, &abort_flag, status, limit_ns, kKernelDebugWait);
}

// ---- host side: tensor maps -------------------------------------------------------------------
}  // namespace

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

int encode_tmap(CUtensorMap *m, bool bf16, int rank, const void *base, const uint64_t *dims,
                const uint64_t *strides_bytes, const uint32_t *box, CUtensorMapSwizzle swz) {
    EncodeTiledFn fn = get_encode();
    if (!fn) return set_error(MOE_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    cuuint64_t gd[3], gs[2];
    cuuint32_t bx[3], es[3] = {1, 1, 1};
    for (int i = 0; i < rank; ++i) {
        gd[i] = dims[i];
        bx[i] = box[i];
    }
    for (int i = 0; i < rank - 1; ++i) gs[i] = strides_bytes[i];
    const CUresult r = fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                          (cuuint32_t)rank, const_cast<void *>(base), gd, gs, bx, es,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return set_error(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return MOE_OK;
}

namespace {

template <bool BF16, bool GATHER, bool GLU, bool SCATTER, bool ROUTER = false, bool BKM = false,
          bool GBWD = false>
int launch_t(const GemmArgs &a, cudaStream_t s) {
    constexpr int EB = BF16 ? 2 : 4;
    constexpr int BK = KBYTES / EB;
    constexpr int CW = KBYTES / EB;
    auto kern = grouped_gemm_kernel<BF16, GATHER, GLU, SCATTER, ROUTER, BKM, GBWD>;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [&] {
        attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)SMEM_BYTES);
    });
    if (attr_err != cudaSuccess)
        return set_error(MOE_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(attr_err));

    CUtensorMap mA, mB0, mB1;
    {
        const uint64_t dims[2] = {(uint64_t)a.K, (uint64_t)a.a_rows};
        const uint64_t str[1] = {(uint64_t)a.K * EB};
        const uint32_t box[2] = {(uint32_t)BK, GATHER ? 1u : (uint32_t)BM};
        int rc = encode_tmap(&mA, BF16, 2, a.A, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
        if (rc) return rc;
    }
    if (BKM) {
        // [E, N, K0] and [E, N, K - K0] with K contiguous, one (BK x BN) box per stage
        const int64_t k0 = a.B1 != nullptr ? a.k_split : a.K;
        if (a.B1 != nullptr && (k0 <= 0 || k0 >= a.K || k0 % BK != 0))
            return set_error(MOE_ERR_UNSUPPORTED, "K split %lld is not a positive multiple of %d "
                             "below K=%lld", (long long)k0, BK, (long long)a.K);
        const uint32_t box[3] = {(uint32_t)BK, (uint32_t)BN, 1u};
        const uint64_t dims0[3] = {(uint64_t)k0, (uint64_t)a.N, (uint64_t)a.E};
        const uint64_t str0[2] = {(uint64_t)k0 * EB, (uint64_t)a.N * k0 * EB};
        int rc = encode_tmap(&mB0, BF16, 3, a.B0, dims0, str0, box, CU_TENSOR_MAP_SWIZZLE_128B);
        if (rc) return rc;
        if (a.B1 != nullptr) {
            const uint64_t dims1[3] = {(uint64_t)(a.K - k0), (uint64_t)a.N, (uint64_t)a.E};
            const uint64_t str1[2] = {(uint64_t)(a.K - k0) * EB, (uint64_t)a.N * (a.K - k0) * EB};
            rc = encode_tmap(&mB1, BF16, 3, a.B1, dims1, str1, box, CU_TENSOR_MAP_SWIZZLE_128B);
            if (rc) return rc;
        } else {
            mB1 = mB0;
        }
    } else {
        const uint64_t dims[3] = {(uint64_t)a.N, (uint64_t)a.K, ROUTER ? 1u : (uint64_t)a.E};
        const uint64_t str[2] = {(uint64_t)a.N * EB, (uint64_t)a.N * a.K * EB};
        const uint32_t box[3] = {(uint32_t)CW, (uint32_t)BK, 1u};
        const CUtensorMapSwizzle swz =
            BF16 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B;
        int rc = encode_tmap(&mB0, BF16, 3, a.B0, dims, str, box, swz);
        if (rc) return rc;
        if (GLU) {
            rc = encode_tmap(&mB1, BF16, 3, a.B1, dims, str, box, swz);
            if (rc) return rc;
        } else {
            mB1 = mB0;
        }
    }
    KParams kp;
    kp.A = a.A;
    kp.K = a.K;
    kp.offsets = a.offsets;
    kp.sorted_rows = a.sorted_rows;
    kp.gates = a.gates;
    kp.out = a.out;
    kp.E = a.E;
    kp.k = a.k;
    kp.N = (int32_t)a.N;
    kp.num_kb = (int32_t)((a.K * EB + KBYTES - 1) / KBYTES);
    constexpr int OUT_COLS = GLU ? BN / 2 : BN;
    kp.n_tiles = (int32_t)((a.N + OUT_COLS - 1) / OUT_COLS);
    kp.S = a.S;
    kp.R = a.R;
    kp.bias = a.bias;
    kp.top_e = a.top_e;
    kp.top_w = a.top_w;
    kp.b_chunks = (int32_t)((a.N + CW - 1) / CW);
    if (ROUTER) {
        kp.stage_bytes = A_BYTES + kp.b_chunks * BK * KBYTES;
        kp.stages = (int32_t)(STAGE_AREA / (size_t)kp.stage_bytes);
        if (kp.stages > MAX_STAGES) kp.stages = MAX_STAGES;
    } else {
        kp.stage_bytes = STAGE_BYTES;
        kp.stages = STAGES;
    }
    kp.k_split = (int32_t)(BKM && a.B1 != nullptr ? a.k_split : a.K + BK);
    kp.a_row_pad = GATHER ? 0 : a.a_row_pad;
    kp.bwd_dh = a.bwd_dh;
    kp.bwd_dw = a.bwd_dw;
    kp.out_row_pad = a.out_row_pad;
    kp.zero_ptr = reinterpret_cast<float4 *>(a.zero_ptr);
    kp.zero_n4 = a.zero_n / 4;
    kp.status = a.status;
    kp.wait_limit_ns = a.wait_limit_ns;
    kern<<<num_sms(), GATHER ? THREADS + GATHER_THREADS : THREADS, SMEM_BYTES, s>>>(mA, mB0, mB1,
                                                                                  kp);
    return MOE_OK;
}

}  // namespace

int launch_grouped_gemm(const GemmArgs &a, cudaStream_t s) {
    // instantiated forms: (gather, glu, scatter) in {(1,1,0), (0,0,1), (1,0,0), (1,0,1),
    // (0,0,0)} x {bf16, f32}, and (0,1,0) in bf16 (SwiGLU on x rows copied to slot order)
    // GLU backward epilogue (bf16, gathered or slot-ordered x, fused gate+up): the MLP backward's
    // recompute
    if (a.glu_bwd) {
        if (a.bf16 && a.glu && !a.scatter && !a.b_kmajor) {
            if (a.gather) return launch_t<true, true, true, false, false, false, true>(a, s);
            return launch_t<true, false, true, false, false, false, true>(a, s);  // slot-ordered x
        }
        return set_error(MOE_ERR_UNSUPPORTED, "GLU backward epilogue form not built");
    }
#define MOE_DISPATCH(BF, G, L, SC)                                                          \
    if (!a.b_kmajor && a.bf16 == BF && a.gather == G && a.glu == L && a.scatter == SC)      \
        return launch_t<BF, G, L, SC>(a, s);
#define MOE_DISPATCH_KM(G, SC)                                                              \
    if (a.b_kmajor && a.bf16 && a.gather == G && !a.glu && a.scatter == SC)                 \
        return launch_t<true, G, false, SC, false, true>(a, s);
    // B K-major (bf16): the input-gradient GEMMs of the backward pass
    MOE_DISPATCH_KM(true, true)
    MOE_DISPATCH_KM(true, false)
    MOE_DISPATCH_KM(false, true)
    MOE_DISPATCH_KM(false, false)
#undef MOE_DISPATCH_KM
    MOE_DISPATCH(true, true, true, false)
    MOE_DISPATCH(true, false, true, false)
    MOE_DISPATCH(true, false, false, true)
    MOE_DISPATCH(true, true, false, false)
    MOE_DISPATCH(true, true, false, true)
    MOE_DISPATCH(true, false, false, false)
    MOE_DISPATCH(false, true, true, false)
    MOE_DISPATCH(false, false, false, true)
    MOE_DISPATCH(false, true, false, false)
    MOE_DISPATCH(false, true, false, true)
    MOE_DISPATCH(false, false, false, false)
#undef MOE_DISPATCH
    return set_error(MOE_ERR_UNSUPPORTED, "grouped GEMM form not built");
}

int launch_route_tc(const void *x, const void *w_gate, const float *bias, int64_t S, int64_t D,
                    int32_t E, int32_t k, int32_t *top_e, float *top_w, unsigned *status,
                    cudaStream_t s) {
    GemmArgs a{};
    a.A = x;
    a.a_rows = S;
    a.B0 = w_gate;  // [D, E] viewed as one expert of a [1, K=D, N=E] weight
    a.B1 = nullptr;
    a.S = S;
    a.R = S;
    a.E = E;
    a.k = k;
    a.K = D;
    a.N = E;
    a.bf16 = true;
    a.bias = bias;
    a.top_e = top_e;
    a.top_w = top_w;
    a.status = status;
    a.wait_limit_ns = kWaitLimitNs;
    // the B map spans one "expert" of [D, E]
    return launch_t<true, false, false, false, true>(a, s);
}

int launch_debug_wait(int64_t limit_ns, unsigned *status, cudaStream_t s) {
    debug_wait_kernel<<<1, 32, 0, s>>>(limit_ns, status);
    return MOE_OK;
}

}  // namespace moe
