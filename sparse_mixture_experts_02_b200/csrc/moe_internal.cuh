// Internal declarations and sm_100a device helpers of the MoE library.
//
// The inline PTX here follows the public PTX ISA (mbarrier, cp.async, cp.async.bulk.tensor,
// tcgen05.alloc / mma / commit / ld / st / fence). No helper here is shared with the CPU oracle.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

// ---- device status word (first 4 bytes of every workspace) ----------------------------------
enum : unsigned {
    kStatusBadExpert = 1u << 0,
    kStatusTimeout = 1u << 1,
    kStatusBadIndex = 1u << 2,  // debug builds: a bounds check skipped an out-of-range index
    // bits 8..15: id of the first kernel whose wait ran out
    kKernelGemm = 1u, kKernelDebugWait = 2u, kKernelAttention = 3u,
};
constexpr size_t kStatusBytes = 256;

// Debug builds (compiled with -DMOE_DEBUG=1, libmoe_b200_debug.so) check every index that a
// kernel reads from its inputs before using it as an address: a gathered token row, a slot, a
// route, the expert offsets behind a tile schedule. An index outside its range sets
// kStatusBadIndex in the status word and the access is skipped; nothing traps. Release builds
// compile the checks away.
#ifndef MOE_DEBUG
#define MOE_DEBUG 0
#endif
constexpr bool kDebugChecks = MOE_DEBUG != 0;

// Default bound of every device-side wait (ns). Kernels here finish in milliseconds; a wait that
// lasts this long means a protocol fault, and the kernel returns instead of hanging the GPU.
constexpr int64_t kWaitLimitNs = 4000000000LL;
// Bound of the teardown waits that drain copies already in flight.
constexpr int64_t kDrainLimitNs = 1000000000LL;

// ---- host-side launchers (defined in the .cu files) -----------------------------------------
int launch_zero_f32(float *p, int64_t n, unsigned *status, cudaStream_t s);
// Returns the number of kernels launched (0 or 1), or -1 after set_error.
int launch_route(const void *x, const void *w_gate, const float *bias, int64_t S, int64_t D,
                 int32_t E, int32_t k, bool bf16, int32_t *top_e, float *top_w, unsigned *status,
                 cudaStream_t s);
size_t map_scratch_bytes(int64_t R, int32_t E);
int launch_sparse_map(const int32_t *top_e, int64_t R, int32_t E, int32_t *counts,
                      int32_t *offsets, int32_t *sparse_rows, int32_t *sorted_rows,
                      int32_t *scratch, unsigned *status, cudaStream_t s, int *n_launch);

struct GemmArgs {
    const void *A;          // gather: x [S, K] token order; else grouped rows [R, K]
    int64_t a_rows;         // S (gather) or R (grouped)
    const void *B0;         // [E, K, N] (gate half for the fused GLU)
    const void *B1;         // [E, K, N] up half (GLU only)
    const int32_t *offsets; // [E+1]
    const int32_t *sorted_rows;  // [R]
    const float *gates;     // [R] by route index, nullable
    void *out;              // grouped [R, N] (dt) or scatter [S, N] f32
    int64_t S, R;
    int32_t E, k;
    int64_t K, N;
    bool bf16, gather, glu, scatter;
    // B K-major (one-CTA kernel, non-GLU): B0 is [E, N, K] with K contiguous (a weight [E, N, K]
    // read as its transpose); with B1 set, B0 covers K indices < k_split ([E, N, k_split]) and
    // B1 the rest ([E, N, K - k_split]); k_split is a multiple of 64 bf16 elements.
    bool b_kmajor;
    int64_t k_split;
    // contiguous A only: slot row p of expert e is read at row p + a_row_pad * e (a padded layout)
    int32_t a_row_pad;
    // GLU backward epilogue (one-CTA kernel, bf16, gathered A, GLU): out is [da | db] bf16 rows
    // of 2N at row p + out_row_pad * e; bwd_dh [R, N] the ungated gradient of h; bwd_dw [R] the
    // route-weight gradient (accumulated atomically, zeroed by the caller); gates = router weights
    bool glu_bwd;
    const void *bwd_dh;
    float *bwd_dw;
    int32_t out_row_pad;
    const float *bias;      // router mode only
    int32_t *top_e;
    float *top_w;
    float *zero_ptr;        // nullable: fp32 buffer (16-byte aligned) the epilogue warps zero
    int64_t zero_n;         // its length (a multiple of 4)
    unsigned *status;
    int64_t wait_limit_ns;
};
int launch_grouped_gemm(const GemmArgs &a, cudaStream_t s);
// Same operation on CTA pairs (tcgen05 cta_group::2, 256-row tiles).
int launch_grouped_gemm_2sm(const GemmArgs &a, cudaStream_t s);
// Picks the two-CTA kernel when experts hold >= 384 rows on average (256-row
// pair tiles waste little there); the environment variable MOE_GEMM_2SM=0/1 forces either kernel.
bool prefer_2sm(int64_t R, int32_t E);
// The choice for the scatter-add forms (GEMM2, the MoA output projection): pairs from 192 rows an
// expert on average.
bool prefer_2sm_scatter(int64_t R, int32_t E);
int launch_debug_wait(int64_t limit_ns, unsigned *status, cudaStream_t s);
// Weight gradient of ParallelLinear: dW[e] = sum over the slots p of expert e of A_p^T (x) dv_p,
// A [a_rows, Din] the source rows in slot order (row stride a_ld elements, 0: Din), dv the
// output-gradient rows in the padded slot layout: expert e's rows start at row offsets[e] + 64 e
// and are followed by zero rows up to the next multiple of 64 (dv_rows >= R + 64 E). dW
// [E, Din, Dout] fp32 is overwritten (zeros for experts without slots). bf16 operands.
struct WgradArgs {
    const void *A;
    int64_t a_rows, a_ld;
    const void *dv;
    int64_t dv_rows, dv_ld;
    const int32_t *offsets; // [E+1]
    int64_t Din, Dout;
    int32_t E;
    float *dW;
    unsigned *status;
    int64_t wait_limit_ns;
};
constexpr int kWgradPad = 64;  // rows of zero padding per expert in the dv layout
int launch_grouped_wgrad(const WgradArgs &a, cudaStream_t s);
// Backward helpers (backward.cu), one warp per slot; Dout a multiple of 8, rows 16-byte aligned.
void launch_cast_bf16(const float *src, void *dst, int64_t n, cudaStream_t s);
// dv[p'] = bf16(gate * dY[row(p)]) with p' = p + 64 e(p) when pad_offsets (the expert offsets)
// is given (the weight gradient's padded layout), else p' = p.
void launch_gate_rows(const void *dY, bool dy_bf16, const int32_t *sorted_rows, const float *gates,
                      int32_t k, int64_t R, int64_t Dout, bool by_token, void *dv,
                      const int32_t *pad_offsets, int32_t E, unsigned *status, cudaStream_t s);
// Zeroes, for every expert, the padding rows after its rows in the padded layout (bf16 rows of
// `cols` elements, row stride ld).
void launch_zero_pad_rows(void *rows, int64_t ld, int64_t cols, const int32_t *offsets, int32_t E,
                          cudaStream_t s);
// xs[p] = x[sorted_rows[p] / k] (bf16 rows of D elements): the slot-ordered rows the weight
// gradient reads by TMA.
void launch_gather_rows(const void *x, const int32_t *sorted_rows, int32_t k, int64_t R, int64_t D,
                        void *xs, unsigned *status, cudaStream_t s);
void launch_rowdot(const void *dY, bool dy_bf16, const void *v, const int32_t *sorted_rows,
                   int32_t k, int64_t R, int64_t Dout, bool by_token, float *dg, unsigned *status,
                   cudaStream_t s);
// (two launches: W_gate^T into w_gate_t [E, D], then the per-token router backward)
void launch_router_bwd(const int32_t *top_e, const float *top_w, const float *dw,
                       const void *w_gate, void *w_gate_t, int64_t S, int64_t D, int32_t E,
                       int32_t k, void *dl, float *dx, int32_t *chunk_offsets, int32_t chunk,
                       int32_t P, cudaStream_t s);
void launch_sum_partials(const float *partial, int64_t n, int32_t P, float *out, cudaStream_t s);
// Router on the tensor cores (bf16, E % 8 == 0): logits of 128-token tiles in TMEM, top-k and
// softmax in the epilogue.
// Attention core of Mixture of Attention: for every route i (token i / k) with slot
// p = sparse_rows[i], o[p] = causal attention of query row q[p] ([R, H*dh] bf16, slot order)
// over the shared keys/values kv [S, 2*H*dh] bf16 (K columns first) up to token i / k. dh is 64
// or 128. Waits are bounded (status word, kernel id kKernelAttention).
int launch_moa_attention(const void *q, const void *kv, const int32_t *sparse_rows, void *o,
                         int64_t R, int64_t S, int32_t H, int32_t dh, int32_t k, unsigned *status,
                         cudaStream_t s);
// Expert parallelism (expert_parallel.cu): pack the routed rows in slot order (row_bytes a
// multiple of 16) with their expert ids; local expert ids of received rows (also clears the
// status word); combine returned fp32 rows per token with the router weights (D % 4 == 0).
void launch_ep_pack(const void *x, size_t row_bytes, const int32_t *top_e,
                    const int32_t *sorted_rows, const int32_t *offsets, int32_t E, int32_t k,
                    int64_t R, void *send, int32_t *send_e, unsigned *status, cudaStream_t s);
void launch_local_ids(const int32_t *ids, int32_t base, int64_t R, int32_t *local,
                      unsigned *status, cudaStream_t s);
void launch_ep_combine(const float *ret, const int32_t *sparse_rows, const float *w, int64_t S,
                       int32_t k, int64_t R, int64_t D, float *out, cudaStream_t s);
// Writes {0, S}: the offsets of one group holding every token.
void launch_kv_offsets(int32_t *off, int64_t S, cudaStream_t s);
int launch_route_tc(const void *x, const void *w_gate, const float *bias, int64_t S, int64_t D,
                    int32_t E, int32_t k, int32_t *top_e, float *top_w, unsigned *status,
                    cudaStream_t s);

// Tiled TMA tensor map (rank 2 or 3) over a bf16 / fp32 tensor; returns MOE_OK or an error.
int encode_tmap(CUtensorMap *m, bool bf16, int rank, const void *base, const uint64_t *dims,
                const uint64_t *strides_bytes, const uint32_t *box, CUtensorMapSwizzle swz);

// error message plumbing (api.cu)
int set_error(int code, const char *fmt, ...);
int num_sms();

}  // namespace moe

// =============================================================================================
// device helpers
// =============================================================================================
#ifdef __CUDACC__
namespace moe {
namespace dev {

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Debug builds: true when 0 <= v < n; otherwise records kStatusBadIndex and returns false.
// Release builds: always true (the check compiles away).
template <typename T>
__device__ __forceinline__ bool debug_in_range(T v, int64_t n, unsigned *status) {
    if constexpr (!kDebugChecks) {
        return true;
    } else {
        if (v >= 0 && (int64_t)v < n) return true;
        if (status != nullptr) atomicOr(status, kStatusBadIndex);
        return false;
    }
}

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---- mbarrier ------------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                     smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase of `bar` with the given parity to complete. Returns false if
// *abort is raised by another role, or if limit_ns passes (then it raises *abort and records a
// timeout in the status word). Never spins forever.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort,
                                          unsigned *status, int64_t limit_ns, unsigned kernel_id) {
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait(a, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(a, parity)) return true;
        if ((it & 63u) == 0) {
            if (abort != nullptr && *abort) return false;
            if ((int64_t)(globaltimer() - t0) > limit_ns) {
                if (abort != nullptr) *abort = 1;
                if (status != nullptr)
                    atomicOr(status, kStatusTimeout | (kernel_id << 8));
                return false;
            }
        }
    }
}

// ---- TMA (cp.async.bulk.tensor) --------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar,
                                            int32_t c0, int32_t c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
        : "memory");
}
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, uint64_t *bar,
                                            int32_t c0, int32_t c1, int32_t c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}
// ---- cp.async (LSU path) ------------------------------------------------------------------------
// 16 bytes global -> shared, bypassing L1; src_bytes = 0 writes zeros (K tail).
__device__ __forceinline__ void cp_async16(uint32_t dst_smem, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst_smem), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}
// One arrival on `bar` once every cp.async this thread issued so far has landed (the barrier's
// expected count must include it: .noinc does not raise the pending count).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.wait_all;" ::: "memory");
}
// Orders this thread's view of generic-proxy shared-memory writes before its later async-proxy
// (tensor core) reads.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---- tcgen05 ---------------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D[tmem] (+)= A[smem desc] x B[smem desc], one instruction, issued by one thread.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// The same with A read from TMEM (M rows = lanes; 16-bit K elements packed two per 32-bit column,
// the lower K index in the low half; one instruction reads K/2 columns from a_tmem).
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void mma_tf32(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive once on `bar` when every tcgen05.mma issued so far by this thread has completed.
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}
// 32 lanes x 32 consecutive 32-bit columns: thread t of the warp gets lane (base lane + t).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// 32 lanes x 32 consecutive 32-bit columns from registers: thread t of the warp writes lane
// (base lane + t).
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ---- shared-memory matrix descriptors (tcgen05 format) -----------------------------------------
// bits [0,14) start>>4, [16,30) LBO>>4, [32,46) SBO>>4, [46,48) version = 1,
// [49,52) base offset = 0, [52] LBO mode = 0, [61,64) layout type:
//   2 = 128-byte swizzle (16-byte units, 8-row / 1024-byte atom),
//   1 = 128-byte swizzle with 32-byte units (4-row / 512-byte atom); the only swizzled layout
//       the tensor cores accept for an MN-major tf32 operand.
constexpr uint32_t kLayoutSw128 = 2;
constexpr uint32_t kLayoutSw128Base32 = 1;
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo,
                                          uint32_t layout) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)(layout & 7u) << 61;
    return d;
}

// Instruction descriptor for kind::f16 (bf16 inputs) / kind::tf32 with f32 accumulation:
// [4,6) D format = 1 (f32); [7,10) A format, [10,13) B format (1 = bf16, 2 = tf32);
// [15] A major (0 = K-major); [16] B major (1 = MN-major); [17,23) N>>3; [24,29) M>>4.
__host__ __device__ constexpr uint32_t idesc_f32acc(bool bf16, uint32_t M, uint32_t N,
                                                     bool b_mn_major, bool a_mn_major = false) {
    return (1u << 4) | ((bf16 ? 1u : 2u) << 7) | ((bf16 ? 1u : 2u) << 10) |
           ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) | ((N >> 3) << 17) |
           ((M >> 4) << 24);
}

// ---- clusters of two CTAs (tcgen05 cta_group::2) ---------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Address of the same shared-memory object in CTA `rank` of the cluster (shared::cluster window).
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
                 ::: "memory");
}
// Arrive on an mbarrier given by its shared::cluster address (possibly in the peer CTA).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
                 : "memory");
}
// Arrive on a barrier of any CTA of the cluster without release ordering. Used only to say
// "this CTA's A rows of a stage are in its own shared memory and fenced for the async proxy":
// in a CTA-pair MMA each SM's tensor core reads its own CTA's A rows, so the signal carries no
// data that another SM must observe. (A release at cluster scope cost ~0.5 us per arrive.)
__device__ __forceinline__ void mbar_arrive_relaxed_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// mbar_wait for barriers that other CTAs of the cluster (or their tensor cores) arrive on.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t *bar, uint32_t parity,
                                                  volatile int *abort, unsigned *status,
                                                  int64_t limit_ns, unsigned kernel_id) {
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait_cluster(a, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait_cluster(a, parity)) return true;
        if ((it & 63u) == 0) {
            if (abort != nullptr && *abort) return false;
            if ((int64_t)(globaltimer() - t0) > limit_ns) {
                if (abort != nullptr) *abort = 1;
                if (status != nullptr) atomicOr(status, kStatusTimeout | (kernel_id << 8));
                return false;
            }
        }
    }
}
__device__ __forceinline__ void tmem_alloc_cg2(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_cg2() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_cg2(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
// One MMA over the CTA pair: M = 256 rows (128 from each CTA's A), N from both CTAs' B halves;
// issued by one thread of the even CTA with descriptors of its own shared memory.
__device__ __forceinline__ void mma_bf16_cg2(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void mma_tf32_cg2(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive once on the barrier at the same offset in every CTA of `cta_mask` when all prior
// tcgen05 operations of this thread have completed.
__device__ __forceinline__ void mma_commit_cg2_mc(uint64_t *bar, uint16_t cta_mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;" ::"r"(smem_u32(bar)),
        "h"(cta_mask)
        : "memory");
}
// TMA tile loads into this CTA's shared memory whose completion is counted on the barrier at
// `bar_cluster` (the even CTA's barrier) - the two-CTA form, no multicast.
__device__ __forceinline__ void tma_load_2d_cg2(void *dst, const CUtensorMap *map,
                                                uint32_t bar_cluster, int32_t c0, int32_t c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1)
        : "memory");
}
__device__ __forceinline__ void tma_load_3d_cg2(void *dst, const CUtensorMap *map,
                                                uint32_t bar_cluster, int32_t c0, int32_t c1,
                                                int32_t c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}
__device__ __forceinline__ void cp_async_commit_group() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ---- vector reduction into global memory ---------------------------------------------------------
__device__ __forceinline__ void red_add_v4(float *addr, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b),
                 "f"(c), "f"(d)
                 : "memory");
}

}  // namespace dev
}  // namespace moe
#endif
