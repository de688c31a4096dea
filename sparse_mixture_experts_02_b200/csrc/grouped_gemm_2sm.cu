// The grouped GEMM on CTA pairs (tcgen05 cta_group::2): each MMA covers a 256-row x 256-column
// tile, 128 rows from each CTA's shared memory, and B split by columns between the two CTAs, so
// each CTA stages only half of B. Per CTA and per 128 bytes of K that is 16 KB of A and 16 KB of
// B (the one-CTA kernel stages 16 + 32 KB for half the MMA work), which halves the operand bytes
// read from shared memory per FLOP and buys six pipeline stages of look-ahead in the same space.
//
// Same forms and sources as the one-CTA kernel (grouped_gemm.cu): the ParallelLinear Core
// Abstraction (ScatterMoE guide, Steps 1-3), its zero-padding tiles per expert ("2. Grouped
// Coordinate Indexing Without Padding"), the fused gate+up SwiGLU GEMM of the TritonMoE abstract.
//
// Roles (both CTAs of a pair run the same tile sequence; the even CTA is the leader):
//   warp 0      TMA producer of this CTA's stage half: its B columns (GLU: the leader loads the
//               128 gate columns, the other CTA the same 128 up columns) and, for contiguous A,
//               its 128 rows; completion is counted on the leader's full barrier.
//   warp 1      TMEM (both CTAs, 2 x 256 columns); in the leader one thread issues the pair
//               MMAs and commits them to the empty / tmem-full barriers of both CTAs.
//   warps 2-5   epilogue of this CTA's 128 accumulator rows (shared code with the one-CTA kernel).
//   warps 6-9   (gathered A) cp.async row gatherers of this CTA's 128 rows; their completion is
//               counted asynchronously (cp.async.mbarrier.arrive.noinc) on a CTA-local barrier.
//   warp 10     (gathered A) relay: waits for each stage's gathered rows of this CTA, makes them
//               visible to the async proxy and arrives on the leader's full barrier, so the MMA
//               issuer waits on one barrier per stage and runs no fence, as with TMA-loaded A.
//               The relay is a thread with no copies of its own in flight, and its arrive is
//               relaxed: a cluster-scope release there measured ~0.5 us a stage, longer than a
//               stage of MMAs, and the proxy fence in the issuer halved the MMA rate.
#include "gemm_common.cuh"

#include <mutex>

namespace moe {
namespace {

using namespace gemm;

constexpr int TM2 = 256;            // rows per pair tile
constexpr int A2_BYTES = 128 * KBYTES;
constexpr int B2_BYTES = 128 * KBYTES;  // this CTA's 128 columns of B
constexpr int STAGE2_BYTES = A2_BYTES + B2_BYTES;
constexpr uint16_t kPairMask = 0x3;
constexpr int RELAY_WARP = (THREADS + GATHER_THREADS) / 32;
constexpr int GATHER_BLOCK = THREADS + GATHER_THREADS + 32;  // threads of a gathered-A CTA

// Shared-memory tail after NS pipeline stages; STG: the scatter epilogue's staging buffers.
template <int NS, bool STG>
struct Smem2T {
    uint64_t full[NS];     // leader: one phase per stage = both CTAs' TMA bytes (+ both relays)
    uint64_t afull[NS];    // both CTAs: this CTA's gathered rows of the stage landed
    uint64_t empty[NS];    // both CTAs: the pair MMAs of the stage are done
    uint64_t tfull[2];     // both CTAs: accumulator b complete
    uint64_t tempty[2];    // leader: both CTAs' epilogues have read accumulator b
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    int32_t off[MAX_E + 1];
    int32_t tstart[MAX_E + 1];
    float stage[STG ? 4 : 1][STG ? 32 * 33 : 1];  // one 32 x 33 buffer per epilogue warp
};
// The SwiGLU form stores h rows straight from registers and needs no staging buffers: it runs a
// seventh stage in their place, with less alignment slack (the kernel checks that the dynamic
// shared memory base needs no more).
template <bool GLU> constexpr int stages2() { return GLU ? 7 : 6; }
template <bool GLU> constexpr size_t slack2() { return GLU ? 768 : 1024; }
template <bool GLU>
constexpr size_t smem2_bytes() {
    return slack2<GLU>() + (size_t)stages2<GLU>() * STAGE2_BYTES +
           sizeof(Smem2T<stages2<GLU>(), !GLU>);
}
static_assert(smem2_bytes<true>() <= 232448 && smem2_bytes<false>() <= 232448,
              "dynamic shared memory per CTA");

// BKM: the weights read K-major ([E, N, K], a weight [E, K, N] of the forward read as its
// transpose, optionally split over two tensor maps at K = k_split), one 64 x 128 box per CTA and
// stage, and slot-ordered A rows in the padded layout (row p of expert e at p + a_row_pad * e):
// the input-gradient GEMMs of the MLP backward. GBWD: the SwiGLU-backward epilogue of the
// recomputed GEMM1 (glu_bwd_row). Both are compile-time forms; the forward's are untouched.
template <bool BF16, bool GATHER, bool GLU, bool SCATTER, bool BKM = false, bool GBWD = false>
__global__ void __cluster_dims__(2, 1, 1)
__launch_bounds__(GATHER ? GATHER_BLOCK : THREADS, 1)
grouped_gemm_2sm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB0,
                        const __grid_constant__ CUtensorMap tmB1, const KParams p) {
    constexpr int EB = BF16 ? 2 : 4;
    constexpr int BK = KBYTES / EB;              // K elements per stage
    constexpr int CW = KBYTES / EB;              // N elements per 128-byte B chunk
    constexpr int NCH = 128 / CW;                // B chunks of this CTA's 128 columns
    constexpr int CHUNK = BK * KBYTES;
    constexpr int B_KSTEP = (32 / EB) * KBYTES;
    constexpr int OUT_COLS = GLU ? BN / 2 : BN;
    static_assert(!BKM || (BF16 && !GLU && !GATHER), "K-major weights: plain bf16 forms");
    static_assert(!GBWD || (BF16 && GLU && !SCATTER && !GATHER), "SwiGLU-backward form");
    constexpr uint32_t IDESC = dev::idesc_f32acc(BF16, 256, BN, !BKM);
    constexpr uint32_t B_LAYOUT = BF16 ? dev::kLayoutSw128 : dev::kLayoutSw128Base32;
    constexpr uint32_t B_SBO = BF16 ? 1024 : 512;
    static_assert(NCH * CHUNK == B2_BYTES, "B half size");

    constexpr int ST2 = stages2<GLU>();
    using Smem2 = Smem2T<ST2, !GLU>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    if ((size_t)(smem - smem_raw) > slack2<GLU>()) {  // uniform over the pair; nothing started
        if (threadIdx.x == 0 && p.status != nullptr)
            atomicOr(p.status, kStatusTimeout | (kKernelGemm << 8));
        return;
    }
    Smem2 &st = *reinterpret_cast<Smem2 *>(smem + (size_t)ST2 * STAGE2_BYTES);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = dev::cluster_ctarank();
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int E = p.E;

    if (threadIdx.x == 0) {
        for (int s = 0; s < ST2; ++s) {
            dev::mbar_init(&st.full[s], GATHER ? 3 : 1);
            dev::mbar_init(&st.afull[s], GATHER_THREADS);
            dev::mbar_init(&st.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            dev::mbar_init(&st.tfull[b], 1);
            dev::mbar_init(&st.tempty[b], 8);
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
        dev::tmem_alloc_cg2(&st.tmem_base, TMEM_COLS);
        dev::tmem_relinquish_cg2();
        dev::tc_fence_before();
    }
    for (int e = threadIdx.x; e <= E; e += blockDim.x) st.off[e] = __ldg(p.offsets + e);
    __syncthreads();
    if (threadIdx.x == 0) {
        build_schedule<TM2>(st.off, st.tstart, E, p.n_tiles);
        debug_check_offsets(st.off, st.tstart, E, p.R, p.status);
    }
    // both CTAs' barriers are initialised before either CTA touches the other's
    dev::cluster_sync();
    dev::tc_fence_after();
    const uint32_t tmem_base = st.tmem_base;
    const int total = st.tstart[E];
    volatile int *abort = &st.abort;

    if (warp == 0) {
        // ------------------------------------------------------------------ TMA producer
        uint32_t s = 0, ph = 0;
        uint32_t issued = 0, last_par = 0;
        bool ok = true;
        const uint32_t tx = 2u * (uint32_t)((GATHER ? 0 : A2_BYTES) + B2_BYTES);
        for (int t = pair; t < total && ok; t += npairs) {
            const TileInfo ti = decode_tile<TM2>(t, st.off, st.tstart, E);
            const int n0 = ti.n_idx * OUT_COLS;
            for (int kb = 0; kb < p.num_kb; ++kb) {
                bool w = true;
                if (lane == 0)
                    w = dev::mbar_wait_cluster(&st.empty[s], ph ^ 1u, abort, p.status,
                                               p.wait_limit_ns, kKernelGemm);
                w = __shfl_sync(0xffffffffu, w, 0);
                if (!w) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    uint8_t *sA = smem + (size_t)s * STAGE2_BYTES;
                    uint8_t *sB = sA + A2_BYTES;
                    const uint32_t full0 = dev::mapa_shared(dev::smem_u32(&st.full[s]), 0);
                    if (leader) dev::mbar_arrive_expect_tx(&st.full[s], tx);
                    const int kc = kb * BK;
                    if (!GATHER) {
                        int arow = ti.row_begin + 128 * (int)rank;
                        if constexpr (BKM) arow += p.a_row_pad * ti.e;
                        dev::tma_load_2d_cg2(sA, &tmA, full0, kc, arow);
                    }
                    if constexpr (BKM) {
                        const bool hi = kc >= p.k_split;
                        dev::tma_load_3d_cg2(sB, hi ? &tmB1 : &tmB0, full0,
                                             hi ? kc - p.k_split : kc, n0 + 128 * (int)rank, ti.e);
                    } else {
#pragma unroll
                        for (int c = 0; c < NCH; ++c) {
                            if (GLU) {
                                dev::tma_load_3d_cg2(sB + c * CHUNK, leader ? &tmB0 : &tmB1, full0,
                                                     n0 + c * CW, kc, ti.e);
                            } else {
                                dev::tma_load_3d_cg2(sB + c * CHUNK, &tmB0, full0,
                                                     n0 + 128 * (int)rank + c * CW, kc, ti.e);
                            }
                        }
                    }
                }
                issued |= 1u << s;
                last_par = (last_par & ~(1u << s)) | (ph << s);
                if (++s == ST2) {
                    s = 0;
                    ph ^= 1u;
                }
            }
        }
        // teardown (leader): every stage issued must have landed in both CTAs before the pair
        // may exit; the other CTA waits at the closing cluster barrier for the leader.
        if (leader && lane == 0) {
            for (int s2 = 0; s2 < ST2; ++s2)
                if (issued & (1u << s2))
                    dev::mbar_wait_cluster(&st.full[s2], (last_par >> s2) & 1u, nullptr, p.status,
                                           kDrainLimitNs, kKernelGemm);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer (leader)
        if (leader && lane == 0) {
            uint32_t s = 0, ph = 0;
            int it = 0;
            bool ok = true;
            for (int t = pair; t < total && ok; t += npairs, ++it) {
                const uint32_t b = it & 1, aph = (it >> 1) & 1;
                if (!dev::mbar_wait_cluster(&st.tempty[b], aph ^ 1u, abort, p.status,
                                            p.wait_limit_ns, kKernelGemm))
                    break;
                dev::tc_fence_after();
                const uint32_t d_tmem = tmem_base + b * BN;
                for (int kb = 0; kb < p.num_kb; ++kb) {
                    if (!dev::mbar_wait_cluster(&st.full[s], ph, abort, p.status, p.wait_limit_ns,
                                                kKernelGemm)) {
                        ok = false;
                        break;
                    }
                    dev::tc_fence_after();
                    const uint32_t sA = dev::smem_u32(smem + (size_t)s * STAGE2_BYTES);
                    const uint32_t sB = sA + A2_BYTES;
#pragma unroll
                    for (int kk = 0; kk < KBYTES / 32; ++kk) {
                        const uint64_t ad =
                            dev::sdesc(sA + kk * 32, 16, 1024, dev::kLayoutSw128);
                        const uint64_t bd =
                            BKM ? dev::sdesc(sB + kk * 32, 16, 1024, dev::kLayoutSw128)
                                : dev::sdesc(sB + kk * B_KSTEP, CHUNK, B_SBO, B_LAYOUT);
                        if (BF16) dev::mma_bf16_cg2(d_tmem, ad, bd, IDESC, (kb | kk) != 0);
                        else dev::mma_tf32_cg2(d_tmem, ad, bd, IDESC, (kb | kk) != 0);
                    }
                    dev::mma_commit_cg2_mc(&st.empty[s], kPairMask);
                    if (++s == ST2) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                dev::mma_commit_cg2_mc(&st.tfull[b], kPairMask);
            }
            // teardown: all pair MMAs complete before TMEM is released
            dev::mma_commit_cg2_mc(&st.drain, 0x1);
            dev::mbar_wait_cluster(&st.drain, 0, nullptr, p.status, kDrainLimitNs, kKernelGemm);
            dev::tc_fence_before();
        }
        __syncwarp();
    } else if (GATHER && warp == RELAY_WARP) {
        // ------------------------------------------------------------------ relay (both CTAs)
        if (lane == 0) {
            uint32_t s = 0, ph = 0;
            bool ok = true;
            for (int t = pair; t < total && ok; t += npairs) {
                for (int kb = 0; kb < p.num_kb; ++kb) {
                    if (!dev::mbar_wait(&st.afull[s], ph, abort, p.status, p.wait_limit_ns,
                                        kKernelGemm)) {
                        ok = false;
                        break;
                    }
                    dev::fence_proxy_async_smem();  // cp.async rows -> tensor core
                    dev::mbar_arrive_relaxed_cluster(
                        dev::mapa_shared(dev::smem_u32(&st.full[s]), 0));
                    if (++s == ST2) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
        }
        __syncwarp();
    } else if (GATHER && warp >= THREADS / 32) {
        // ------------------------------------------------------------------ row gatherers
        const int gw = warp - THREADS / 32;
        const int chunk = lane & 7;
        const int rsub = lane >> 3;
        const int64_t row_bytes = (int64_t)p.K * EB;
        const uint8_t *xa = reinterpret_cast<const uint8_t *>(p.A);
        // sorted_rows entries of this thread's 8 rows of tile t (tail rows repeat a valid row)
        auto fetch_rows = [&](int t, int *ent) {
            const TileInfo ti = decode_tile<TM2>(t, st.off, st.tstart, E);
            const int rbeg = ti.row_begin + 128 * (int)rank;
            const int rows = min(128, ti.rows - 128 * (int)rank);  // may be <= 0
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int r = gw * 32 + i * 4 + rsub;
                ent[i] = rows > 0 ? __ldg(p.sorted_rows + rbeg + min(r, rows - 1)) : 0;
            }
        };
        // x row pointers of tile t from its entries; returns this CTA's rows of it (may be <= 0)
        auto row_ptrs = [&](int t, const int *ent, const uint8_t **src) {
            const TileInfo ti = decode_tile<TM2>(t, st.off, st.tstart, E);
            const int rows = min(128, ti.rows - 128 * (int)rank);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                // debug builds: a route outside [0, S*k) reads row 0 instead (and is flagged)
                const int en = rows > 0 && dev::debug_in_range(ent[i], (int64_t)p.S * p.k, p.status)
                                   ? ent[i] : 0;
                src[i] = xa + (int64_t)(en / p.k) * row_bytes;
            }
            return rows;
        };
        // Shared memory is saturated by the tensor core, so a tile's schedule lookups, index
        // loads and divisions take ~2 us: the next tile's pointers are formed after the current
        // tile's second stage is issued, and its entries are loaded a tile earlier still, so
        // nothing but a register swap sits between two tiles' copies.
        int ent[8];
        const uint8_t *src[8], *nsrc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) src[i] = nsrc[i] = xa;
        int rows = 0, nrows = 0;
        if (pair < total) {
            fetch_rows(pair, ent);
            rows = row_ptrs(pair, ent, src);
            if (pair + npairs < total) fetch_rows(pair + npairs, ent);
        }
        const int prep_kb = min(1, p.num_kb - 1);
        uint32_t s = 0, ph = 0;
        bool ok = true;
        for (int t = pair; t < total && ok; t += npairs) {
            for (int kb = 0; kb < p.num_kb; ++kb) {
                bool w = true;
                if (lane == 0)
                    w = dev::mbar_wait_cluster(&st.empty[s], ph ^ 1u, abort, p.status,
                                               p.wait_limit_ns, kKernelGemm);
                w = __shfl_sync(0xffffffffu, w, 0);
                if (!w) {
                    ok = false;
                    break;
                }
                const uint32_t sA = dev::smem_u32(smem + (size_t)s * STAGE2_BYTES);
                const int64_t cb = (int64_t)kb * KBYTES + chunk * 16;
                const uint32_t nbytes = cb < row_bytes ? 16u : 0u;  // zero-fill past K
                // rows past this CTA's share are not copied: an A row only feeds its own output
                // row, which the epilogue discards
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = gw * 32 + i * 4 + rsub;
                    const uint32_t dst = sA + r * KBYTES + ((chunk ^ (r & 7)) << 4);
                    if (r < rows) dev::cp_async16(dst, nbytes ? src[i] + cb : src[i], nbytes);
                }
                dev::cp_async_arrive_noinc(&st.afull[s]);
                if (kb == prep_kb && t + npairs < total) {
                    nrows = row_ptrs(t + npairs, ent, nsrc);
                    if (t + 2 * npairs < total) fetch_rows(t + 2 * npairs, ent);
                }
                if (++s == ST2) {
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
        const int q = warp & 3;
        const int r = q * 32 + lane;
        const uint32_t tempty0_base = dev::mapa_shared(dev::smem_u32(&st.tempty[0]), 0);
        int it = 0;
        for (int t = pair; t < total; t += npairs, ++it) {
            const TileInfo ti = decode_tile<TM2>(t, st.off, st.tstart, E);
            const uint32_t b = it & 1, aph = (it >> 1) & 1;
            bool w = true;
            if (lane == 0)
                w = dev::mbar_wait_cluster(&st.tfull[b], aph, abort, p.status, p.wait_limit_ns,
                                           kKernelGemm);
            w = __shfl_sync(0xffffffffu, w, 0);
            if (!w) break;
            dev::tc_fence_after();
            const int rows = ti.rows - 128 * (int)rank;
            const int prow = ti.row_begin + 128 * (int)rank + r;
            bool valid = r < rows && prow >= 0 && prow < p.R;
            int64_t orow = prow;
            float g = 1.0f;
            if (valid && (SCATTER || p.gates != nullptr)) {
                const int i = __ldg(p.sorted_rows + prow);
                if (SCATTER) orow = i / p.k;
                if (p.gates != nullptr && i >= 0 && i < p.R) g = __ldg(p.gates + i);
                if (!dev::debug_in_range(i, p.R, p.status) || i < 0 || i >= p.R) valid = false;
            }
            const int n0 = ti.n_idx * OUT_COLS;
            const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + b * BN;
            if constexpr (GBWD) {
                const int64_t route = valid ? (int64_t)__ldg(p.sorted_rows + prow) : 0;
                glu_bwd_row(p, tbase, valid, prow, route, g,
                            prow + (int64_t)p.out_row_pad * ti.e, n0);
            } else if constexpr (GLU) {
                epilogue_row<BF16, GLU, SCATTER>(p, tbase, valid, orow, g, n0, nullptr);
            } else {
                epilogue_row<BF16, GLU, SCATTER>(p, tbase, valid, orow, g, n0, st.stage[q]);
            }
            dev::tc_fence_before();
            __syncwarp();
            if (lane == 0) dev::mbar_arrive_cluster(tempty0_base + b * (uint32_t)sizeof(uint64_t));
        }
    }

    __syncthreads();
    dev::cluster_sync();
    if (warp == 1) {
        dev::tc_fence_after();
        dev::tmem_dealloc_cg2(tmem_base, TMEM_COLS);
    }
}

template <bool BF16, bool GATHER, bool GLU, bool SCATTER, bool BKM = false, bool GBWD = false>
int launch_2sm_t(const GemmArgs &a, cudaStream_t s, int n_pairs) {
    constexpr int EB = BF16 ? 2 : 4;
    constexpr int BK = KBYTES / EB;
    constexpr int CW = KBYTES / EB;
    auto kern = grouped_gemm_2sm_kernel<BF16, GATHER, GLU, SCATTER, BKM, GBWD>;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [&] {
        attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)smem2_bytes<GLU>());
    });
    if (attr_err != cudaSuccess)
        return set_error(MOE_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(attr_err));
    CUtensorMap mA, mB0, mB1;
    {
        const uint64_t dims[2] = {(uint64_t)a.K, (uint64_t)a.a_rows};
        const uint64_t str[1] = {(uint64_t)a.K * EB};
        const uint32_t box[2] = {(uint32_t)BK, 128u};
        int rc = encode_tmap(&mA, BF16, 2, a.A, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
        if (rc) return rc;
    }
    if (BKM) {
        // [E, N, K0] and [E, N, K - K0] with K contiguous, one (BK x 128) box per CTA and stage
        const int64_t k0 = a.B1 != nullptr ? a.k_split : a.K;
        if (a.B1 != nullptr && (k0 <= 0 || k0 >= a.K || k0 % BK != 0))
            return set_error(MOE_ERR_UNSUPPORTED, "K split %lld is not a positive multiple of %d "
                             "below K=%lld", (long long)k0, BK, (long long)a.K);
        const uint32_t box[3] = {(uint32_t)BK, 128u, 1u};
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
        const uint64_t dims[3] = {(uint64_t)a.N, (uint64_t)a.K, (uint64_t)a.E};
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
    KParams kp{};
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
    kp.zero_ptr = reinterpret_cast<float4 *>(a.zero_ptr);
    kp.zero_n4 = a.zero_n / 4;
    kp.status = a.status;
    kp.wait_limit_ns = a.wait_limit_ns;
    kp.k_split = (int32_t)(BKM && a.B1 != nullptr ? a.k_split : a.K + BK);
    kp.a_row_pad = BKM ? a.a_row_pad : 0;
    kp.out_row_pad = a.out_row_pad;
    kp.bwd_dh = a.bwd_dh;
    kp.bwd_dw = a.bwd_dw;
    kern<<<2 * n_pairs, GATHER ? GATHER_BLOCK : THREADS, smem2_bytes<GLU>(), s>>>(mA, mB0, mB1,
                                                                              kp);
    return MOE_OK;
}

// Pairs of CTAs that fit on the device at once (a persistent grid larger than that would
// serialise whole pairs behind each other).
int max_pairs() {
    static int cached[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && cached[dev] > 0) return cached[dev];
    int pairs = num_sms() / 2;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(2 * pairs);
    cfg.blockDim = dim3(GATHER_BLOCK);
    cfg.dynamicSmemBytes = smem2_bytes<true>();
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    auto kern = grouped_gemm_2sm_kernel<true, true, true, false>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem2_bytes<true>());
    if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) == cudaSuccess && clusters > 0 &&
        clusters < pairs)
        pairs = clusters;
    cudaGetLastError();
    if (dev >= 0 && dev < 64) cached[dev] = pairs;
    return pairs;
}

}  // namespace

int launch_grouped_gemm_2sm(const GemmArgs &a, cudaStream_t s) {
    const int pairs = max_pairs();
    // the MLP backward's forms: SwiGLU-backward epilogue on slot-ordered x; K-major weights on
    // slot-ordered (padded) rows, into slot order or scatter-added into tokens
    if (a.glu_bwd) {
        if (a.bf16 && !a.gather && a.glu && !a.scatter && !a.b_kmajor && a.a_row_pad == 0)
            return launch_2sm_t<true, false, true, false, false, true>(a, s, pairs);
        return set_error(MOE_ERR_UNSUPPORTED, "two-CTA GLU backward form not built");
    }
    if (a.b_kmajor) {
        if (a.bf16 && !a.gather && !a.glu)
            return a.scatter ? launch_2sm_t<true, false, false, true, true, false>(a, s, pairs)
                             : launch_2sm_t<true, false, false, false, true, false>(a, s, pairs);
        return set_error(MOE_ERR_UNSUPPORTED, "two-CTA K-major B form not built");
    }
    if (a.a_row_pad != 0)
        return set_error(MOE_ERR_UNSUPPORTED, "two-CTA grouped GEMM: padded A without K-major B");
#define MOE_DISPATCH2(BF, G, L, SC)                                                         \
    if (a.bf16 == BF && a.gather == G && a.glu == L && a.scatter == SC)                     \
        return launch_2sm_t<BF, G, L, SC>(a, s, pairs);
    MOE_DISPATCH2(true, true, true, false)
    MOE_DISPATCH2(true, false, true, false)
    MOE_DISPATCH2(true, false, false, true)
    MOE_DISPATCH2(true, true, false, false)
    MOE_DISPATCH2(true, true, false, true)
    MOE_DISPATCH2(true, false, false, false)
    MOE_DISPATCH2(false, true, true, false)
    MOE_DISPATCH2(false, false, false, true)
    MOE_DISPATCH2(false, true, false, false)
    MOE_DISPATCH2(false, true, false, true)
    MOE_DISPATCH2(false, false, false, false)
#undef MOE_DISPATCH2
    return set_error(MOE_ERR_UNSUPPORTED, "two-CTA grouped GEMM form not built");
}

}  // namespace moe
