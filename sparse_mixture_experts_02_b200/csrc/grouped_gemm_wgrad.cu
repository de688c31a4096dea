// Weight gradient of ParallelLinear on the sm_100a tensor cores: for every expert e,
//   dW[e] = sum over the slots p of e of  A_p^T (x) dv_p        ([Din, Dout], fp32)
// with A_p the input row of slot p and dv_p its gated output-gradient row. The reduction runs
// over an expert's slots, so the K extent of a tile is that expert's row count: any value, zero
// included.
//
// Source: ScatterMoE guide, "3. Fused Backward Pass Dynamics" (the weight gradient of expert e
// accumulates the outer products of its tokens' inputs and gated output gradients). The guide
// reduces inside shared memory to avoid global atomics; here each output tile is owned by one CTA
// and reduced in TMEM over the expert's slots, so no atomics are needed either.
//
// Operands (both MN-major: the K index, a slot, is the row): A in slot order, dv in a padded
// slot order where expert e's rows start at offsets[e] + 64 e and are followed by zero rows up
// to the next multiple of 64. A stage of 64 slots may run past the expert's last slot; those A
// rows belong to the next expert, but their dv rows are zero, so they add nothing. Both come by
// TMA (cp.async gathers of A cost ~40% here: the epilogue already loads the LSU path).
//
// Design (one CTA per SM, persistent):
//   warp 0     TMA producer: per stage 64 A rows x 128 columns (2 boxes of 64 x 64) and 64 dv
//              rows x 256 columns (4 boxes), 128-byte swizzle.
//   warp 1     TMEM owner (two 128 x 256 fp32 accumulators) and MMA issuer: 4 MMAs of M=128
//              (Din), N=256 (Dout), K=16 rows per stage.
//   warps 2-5  epilogue: accumulator lane m -> dW[e][m0 + m][n0 .. n0 + 255], staged through
//              shared memory in 32 x 32 chunks so each store covers 4 rows x 128 bytes; a tile of
//              an expert without slots stores zeros.
// Tiles are (expert, N tile, M tile), expert-major. Every wait is bounded (mbar_wait).
#include "gemm_common.cuh"

#include <mutex>

namespace moe {
namespace {

using namespace gemm;

constexpr int WK = 64;                     // slots (K rows) per stage
constexpr int WCH = 64 * KBYTES;           // one 64-column chunk of a stage: 64 rows x 128 B
constexpr int WA_BYTES = 2 * WCH;          // A: 128 columns of Din
constexpr int WB_BYTES = 4 * WCH;          // B: 256 columns of Dout
static_assert(WA_BYTES == A_BYTES && WB_BYTES == B_BYTES, "stage layout of the forward kernel");

struct WParams {
    const int32_t *offsets;
    int64_t Din, Dout;
    int32_t E;
    float *dW;
    int32_t m_tiles, n_tiles;
    unsigned *status;
    int64_t wait_limit_ns;
};

__device__ __forceinline__ void wtile(int t, int per_e, int m_tiles, int &e, int &n, int &m) {
    e = t / per_e;
    const int local = t - e * per_e;
    n = local / m_tiles;
    m = local - n * m_tiles;
}

__global__ void __launch_bounds__(THREADS, 1)
grouped_wgrad_kernel(const __grid_constant__ CUtensorMap tmA,
                     const __grid_constant__ CUtensorMap tmB, const WParams p) {
    constexpr uint32_t IDESC = dev::idesc_f32acc(true, BM, BN, true, true);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    SmemTail &st = *reinterpret_cast<SmemTail *>(smem + STAGE_AREA);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = p.E;
    const int per_e = p.m_tiles * p.n_tiles;
    const int total = E * per_e;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            dev::mbar_init(&st.full[s], 1);
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
        dev::prefetch_tmap(&tmB);
    }
    if (warp == 1) {
        dev::tmem_alloc(&st.tmem_base, TMEM_COLS);
        dev::tmem_relinquish();
        dev::tc_fence_before();
    }
    for (int e = threadIdx.x; e <= E; e += blockDim.x) st.off[e] = __ldg(p.offsets + e);
    __syncthreads();
    dev::tc_fence_after();
    const uint32_t tmem_base = st.tmem_base;
    volatile int *abort = &st.abort;

    if (warp == 0) {
        // ------------------------------------------------------------------ TMA producer (B)
        uint32_t s = 0, ph = 0, issued = 0, last_par = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
            int e, n, m;
            wtile(t, per_e, p.m_tiles, e, n, m);
            const int r0 = st.off[e], nkb = (st.off[e + 1] - r0 + WK - 1) / WK;
            for (int kb = 0; kb < nkb; ++kb) {
                bool w = true;
                if (lane == 0)
                    w = dev::mbar_wait(&st.empty[s], ph ^ 1u, abort, p.status, p.wait_limit_ns,
                                       kKernelGemm);
                w = __shfl_sync(0xffffffffu, w, 0);
                if (!w) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    uint8_t *sA = smem + (size_t)s * STAGE_BYTES;
                    uint8_t *sB = sA + WA_BYTES;
                    dev::mbar_arrive_expect_tx(&st.full[s], (uint32_t)(WA_BYTES + WB_BYTES));
#pragma unroll
                    for (int c = 0; c < 2; ++c)
                        dev::tma_load_2d(sA + c * WCH, &tmA, &st.full[s], m * BM + c * 64,
                                         r0 + kb * WK);
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        dev::tma_load_2d(sB + c * WCH, &tmB, &st.full[s], n * BN + c * 64,
                                         r0 + kWgradPad * e + kb * WK);
                }
                issued |= 1u << s;
                last_par = (last_par & ~(1u << s)) | (ph << s);
                if (++s == STAGES) {
                    s = 0;
                    ph ^= 1u;
                }
            }
        }
        if (lane == 0) {
            for (int s2 = 0; s2 < STAGES; ++s2)
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
                int e, n, m;
                wtile(t, per_e, p.m_tiles, e, n, m);
                const int nkb = (st.off[e + 1] - st.off[e] + WK - 1) / WK;
                const uint32_t b = it & 1, aph = (it >> 1) & 1;
                if (!dev::mbar_wait(&st.tempty[b], aph ^ 1u, abort, p.status, p.wait_limit_ns,
                                    kKernelGemm))
                    break;
                dev::tc_fence_after();
                const uint32_t d_tmem = tmem_base + b * BN;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!dev::mbar_wait(&st.full[s], ph, abort, p.status, p.wait_limit_ns,
                                        kKernelGemm)) {
                        ok = false;
                        break;
                    }
                    dev::tc_fence_after();
                    const uint32_t sA = dev::smem_u32(smem + (size_t)s * STAGE_BYTES);
                    const uint32_t sB = sA + WA_BYTES;
#pragma unroll
                    for (int kk = 0; kk < WK / 16; ++kk) {
                        // 16 K rows per MMA: 16 lines of 128 B into every 64-column chunk
                        const uint64_t ad =
                            dev::sdesc(sA + kk * 16 * KBYTES, WCH, 1024, dev::kLayoutSw128);
                        const uint64_t bd =
                            dev::sdesc(sB + kk * 16 * KBYTES, WCH, 1024, dev::kLayoutSw128);
                        dev::mma_bf16(d_tmem, ad, bd, IDESC, (kb | kk) != 0);
                    }
                    dev::mma_commit(&st.empty[s]);
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                dev::mma_commit(&st.tfull[b]);  // also for a tile without slots (nothing pending)
            }
            dev::mma_commit(&st.drain);
            dev::mbar_wait(&st.drain, 0, nullptr, p.status, kDrainLimitNs, kKernelGemm);
            dev::tc_fence_before();
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------------ epilogue
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        int it = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x, ++it) {
            int e, n, m;
            wtile(t, per_e, p.m_tiles, e, n, m);
            const bool empty_e = st.off[e + 1] == st.off[e];
            const uint32_t b = it & 1, aph = (it >> 1) & 1;
            bool w = true;
            if (lane == 0)
                w = dev::mbar_wait(&st.tfull[b], aph, abort, p.status, p.wait_limit_ns,
                                   kKernelGemm);
            w = __shfl_sync(0xffffffffu, w, 0);
            if (!w) break;
            dev::tc_fence_after();
            // Each 32 x 32 chunk of the warp's rows goes through shared memory (row stride 33
            // floats), so a store instruction covers 4 rows x 128 contiguous bytes of dW instead
            // of 16 bytes in each of 32 rows: the weight gradient writes 16x more bytes per FLOP
            // than the forward GEMMs.
            float *stg = st.stage[q];
            const int rsub = lane >> 3, cc = (lane & 7) * 4;
            const int64_t row0 = (int64_t)m * BM + q * 32;  // first dW[e] row of this warp
            float *dWe = p.dW + (int64_t)e * p.Din * p.Dout;
            const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + b * BN;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                const int64_t col0 = (int64_t)n * BN + c * 32;
                if (col0 >= p.Dout) break;  // warp-uniform
                uint32_t v[32];
                if (!empty_e) {
                    dev::tmem_ld32(tbase + c * 32, v);
                    dev::tmem_ld_wait();
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = 0u;
                }
#pragma unroll
                for (int j = 0; j < 32; ++j) stg[lane * 33 + j] = __uint_as_float(v[j]);
                __syncwarp();
#pragma unroll
                for (int pass = 0; pass < 8; ++pass) {
                    const int rr = pass * 4 + rsub;
                    const int64_t grow = row0 + rr;
                    if (grow < p.Din && col0 + cc < p.Dout) {
                        const float *sv = stg + rr * 33 + cc;
                        *reinterpret_cast<float4 *>(dWe + grow * p.Dout + col0 + cc) =
                            make_float4(sv[0], sv[1], sv[2], sv[3]);
                    }
                }
                __syncwarp();
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

}  // namespace

int launch_grouped_wgrad(const WgradArgs &a, cudaStream_t s) {
    const int64_t m_tiles = (a.Din + BM - 1) / BM, n_tiles = (a.Dout + BN - 1) / BN;
    if (a.a_rows <= 0 || a.E <= 0) {
        // no slot at all: every expert's gradient is zero
        launch_zero_f32(a.dW, (int64_t)a.E * a.Din * a.Dout, nullptr, s);
        return MOE_OK;
    }
    if ((int64_t)a.E * m_tiles * n_tiles >= (int64_t(1) << 31))
        return set_error(MOE_ERR_UNSUPPORTED, "weight-gradient tile count too large");
    auto kern = grouped_wgrad_kernel;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [&] {
        attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)SMEM_BYTES);
    });
    if (attr_err != cudaSuccess)
        return set_error(MOE_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(attr_err));
    CUtensorMap mA, mB;
    {
        const uint64_t dims[2] = {(uint64_t)a.Din, (uint64_t)a.a_rows};
        const uint64_t str[1] = {(uint64_t)(a.a_ld > 0 ? a.a_ld : a.Din) * 2};
        const uint32_t box[2] = {64u, (uint32_t)WK};
        int rc = encode_tmap(&mA, true, 2, a.A, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
        if (rc) return rc;
    }
    {
        const uint64_t dims[2] = {(uint64_t)a.Dout, (uint64_t)a.dv_rows};
        const uint64_t str[1] = {(uint64_t)(a.dv_ld > 0 ? a.dv_ld : a.Dout) * 2};
        const uint32_t box[2] = {64u, (uint32_t)WK};
        int rc = encode_tmap(&mB, true, 2, a.dv, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
        if (rc) return rc;
    }
    WParams wp;
    wp.offsets = a.offsets;
    wp.Din = a.Din;
    wp.Dout = a.Dout;
    wp.E = a.E;
    wp.dW = a.dW;
    wp.m_tiles = (int32_t)m_tiles;
    wp.n_tiles = (int32_t)n_tiles;
    wp.status = a.status;
    wp.wait_limit_ns = a.wait_limit_ns;
    kern<<<num_sms(), THREADS, SMEM_BYTES, s>>>(mA, mB, wp);
    return MOE_OK;
}

}  // namespace moe
