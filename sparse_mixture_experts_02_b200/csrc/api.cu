// C ABI of the MoE library: argument checks, workspace layout, launch order, status reporting.
// Every public call validates on the host, then enqueues kernels on the caller's stream; nothing
// here synchronises except moe_check_device_status.
#include "moe_internal.cuh"

#include <stdarg.h>
#include <stdlib.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

namespace moe {

static thread_local char g_err[512] = "";
static thread_local int g_launches = 0;
static thread_local void *g_prof_events[8] = {};
static thread_local int g_prof_n = 0;

int set_error(int code, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return code;
}

// True when the environment variable is set to "0" (switches for tests and paired timings).
bool env_off(const char *name) {
    const char *v = getenv(name);
    return v != nullptr && v[0] == '0';
}

bool prefer_2sm(int64_t R, int32_t E) {
    const char *env = getenv("MOE_GEMM_2SM");
    if (env != nullptr && (env[0] == '0' || env[0] == '1')) return env[0] == '1';
    // Pair tiles pay off, for gathered and slot-ordered A alike, when experts are long enough
    // that the 256-row tiles waste little (measured: ~1024 and ~1536 rows an expert gain 5-7% on
    // a forward; ~256 rows an expert lose 5%, ~32 lose 25%).
    return E > 0 && R / E >= 384;
}

// The same choice for the scatter-add forms (h rows by TMA, fp32 reductions into tokens): pairs
// pay off from fewer rows an expert there (measured at ~256 rows: GEMM2 0.730 -> 0.686 ms on
// pairs, where the fused gate+up GEMM1 loses 7%; at ~32 rows both lose).
bool prefer_2sm_scatter(int64_t R, int32_t E) {
    const char *env = getenv("MOE_GEMM_2SM");
    if (env != nullptr && (env[0] == '0' || env[0] == '1')) return env[0] == '1';
    return E > 0 && R / E >= 192;
}

int num_sms() {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 1;
}

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Supported device: compute capability 10.0 (checked once per device).
int check_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return set_error(MOE_ERR_CUDA, "cudaGetDevice failed");
    static std::mutex mu;
    static int known[64] = {0};  // 0 unknown, 1 ok, -1 unsupported
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= 64) return set_error(MOE_ERR_UNSUPPORTED, "device index %d", dev);
    if (known[dev] == 0) {
        int major = 0, minor = 0;
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        known[dev] = (major == 10 && minor == 0) ? 1 : -1;
    }
    if (known[dev] < 0)
        return set_error(MOE_ERR_UNSUPPORTED, "this library is built for sm_100a (B200) only");
    return MOE_OK;
}

int check_launch(const char *what) {
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(MOE_ERR_CUDA, "%s launch: %s", what, cudaGetErrorString(e));
    return MOE_OK;
}

int check_dims(int64_t S, int32_t E, int32_t k) {
    if (S < 0) return set_error(MOE_ERR_INVALID_ARG, "S must be >= 0 (got %lld)", (long long)S);
    if (E < 1 || E > 256) return set_error(MOE_ERR_INVALID_ARG, "E must be in [1, 256] (got %d)", E);
    if (k < 1 || k > 8 || k > E)
        return set_error(MOE_ERR_INVALID_ARG, "k must be in [1, min(E, 8)] (got k=%d, E=%d)", k, E);
    if (S * (int64_t)k >= (int64_t(1) << 31))
        return set_error(MOE_ERR_INVALID_ARG, "S*k must be < 2^31");
    return MOE_OK;
}

int check_feat(const char *name, int64_t v) {
    if (v <= 0 || v % 8 != 0 || v >= (int64_t(1) << 31))
        return set_error(MOE_ERR_INVALID_ARG, "%s must be a positive multiple of 8 below 2^31 (got %lld)",
                         name, (long long)v);
    return MOE_OK;
}

int check_ptr(const char *name, const void *p, size_t align, bool nullable = false) {
    if (p == nullptr) {
        if (nullable) return MOE_OK;
        return set_error(MOE_ERR_INVALID_ARG, "%s is null", name);
    }
    if (!aligned(p, align)) return set_error(MOE_ERR_INVALID_ARG, "%s is not %zu-byte aligned", name, align);
    return MOE_OK;
}

int check_dtype(moe_dtype dt) {
    if (dt != MOE_F32 && dt != MOE_BF16) return set_error(MOE_ERR_UNSUPPORTED, "unknown dtype %d", (int)dt);
    return MOE_OK;
}

size_t esize(moe_dtype dt) { return dt == MOE_BF16 ? 2 : 4; }

// ---- workspace layout ------------------------------------------------------------------------
struct MlpLayout {
    size_t status, top_e, top_w, counts, offsets, sparse_rows, sorted_rows, scratch, h, xs,
        xs_bytes, total;
};

// Whether the forward copies the x rows to slot order before GEMM1 (decided by the shapes alone,
// so that the workspace size never depends on the environment). The copy costs 4 R D bytes of
// HBM traffic; GEMM1 on TMA-loaded rows instead of rows gathered on load saved ~10% of its time
// on CTA pairs (experts of >= 384 rows), which outweighs the copy once F >= 2048 (7.5% of the
// Mixtral-shaped prefill forward, F = 14336; no gain at F = 1408).
bool pregather_shape(int64_t R, int64_t D, int64_t F, int32_t E, moe_dtype dt) {
    return dt == MOE_BF16 && E > 0 && D > 0 && R / E >= 384 && F >= 2048;
}

// with_xs: the MoE forward's layout (x rows in slot order after h when pregather_shape holds);
// the expert-parallel forward, which gathers its received rows on load, has none.
MlpLayout mlp_layout(int64_t S, int64_t D, int64_t F, int32_t E, int32_t k, moe_dtype dt,
                     bool with_xs = true) {
    const int64_t R = S * k;
    MlpLayout L;
    size_t o = 0;
    L.status = o; o += kStatusBytes;
    L.top_e = o; o = align_up(o + sizeof(int32_t) * (size_t)R);
    L.top_w = o; o = align_up(o + sizeof(float) * (size_t)R);
    L.counts = o; o = align_up(o + sizeof(int32_t) * (size_t)E);
    L.offsets = o; o = align_up(o + sizeof(int32_t) * (size_t)(E + 1));
    L.sparse_rows = o; o = align_up(o + sizeof(int32_t) * (size_t)R);
    L.sorted_rows = o; o = align_up(o + sizeof(int32_t) * (size_t)R);
    L.scratch = o; o = align_up(o + map_scratch_bytes(R, E));
    L.h = o; o = align_up(o + esize(dt) * (size_t)R * (size_t)F);
    L.xs_bytes = with_xs && pregather_shape(R, D, F, E, dt) ? esize(dt) * (size_t)R * (size_t)D : 0;
    L.xs = o; o = align_up(o + L.xs_bytes);
    L.total = o;
    return L;
}

// Mixture of Attention forward: the routing prefix of the MLP layout (identical offsets, so the
// routing views of an "mlp_forward" workspace apply), then the one-group offsets of the shared
// key/value projection, kv [S, 2 HD], q and the attention output o ([R, HD] each, slot order),
// all bf16.
struct MoaLayout {
    MlpLayout base;
    size_t kv_off, kv, q, o, total;
};

MoaLayout moa_layout(int64_t S, int64_t HD, int32_t E, int32_t k) {
    const int64_t R = S * k;
    MoaLayout L;
    L.base = mlp_layout(S, 0, 0, E, k, MOE_BF16);
    size_t o = L.base.total;
    L.kv_off = o; o = align_up(o + 2 * sizeof(int32_t));
    L.kv = o; o = align_up(o + 2 * (size_t)S * 2 * (size_t)HD);
    L.q = o; o = align_up(o + 2 * (size_t)R * (size_t)HD);
    L.o = o; o = align_up(o + 2 * (size_t)R * (size_t)HD);
    L.total = o;
    return L;
}

// ParallelLinear backward scratch: status, bf16 copy of an fp32 dY [S, Dout], gated rows dv in
// the weight gradient's padded layout [R + 64 E, Dout] bf16, x rows in slot order [R, Din] (for
// gathered inputs), ungated forward rows v [R, Dout] bf16 (gate gradient).
struct BwdLayout {
    size_t status, dyb, dv, xs, v, total;
};

BwdLayout bwd_layout(int64_t S, int64_t Din, int64_t Dout, int32_t E, int32_t k) {
    const int64_t R = S * k;
    BwdLayout L;
    size_t o = 0;
    L.status = o; o += kStatusBytes;
    L.dyb = o; o = align_up(o + 2 * (size_t)S * (size_t)Dout);
    L.dv = o; o = align_up(o + 2 * (size_t)(R + (int64_t)kWgradPad * E) * (size_t)Dout);
    L.xs = o; o = align_up(o + 2 * (size_t)R * (size_t)Din);
    L.v = o; o = align_up(o + 2 * (size_t)R * (size_t)Dout);
    L.total = o;
    return L;
}

// The W_gate gradient reduces over all S tokens in one "expert": split into P chunks of
// consecutive tokens (at least 256 each) so that about 296 tiles (two per SM) run, then summed.
int32_t router_chunks(int64_t S, int64_t D) {
    const int64_t m_tiles = (D + 127) / 128;
    int64_t P = (296 + m_tiles - 1) / m_tiles;
    const int64_t by_rows = (S + 255) / 256;
    if (P > by_rows) P = by_rows;
    if (P > 256) P = 256;  // the weight-gradient kernel holds at most 256 "experts"
    return (int32_t)(P < 1 ? 1 : P);
}

// MLP backward scratch (the forward's workspace supplies routing, map and h).
struct MlpBwdLayout {
    size_t status, dhp, dpre, dw, dv, dl, xs, off1, partial, wgt, total;
};

MlpBwdLayout mlp_bwd_layout(int64_t S, int64_t D, int64_t F, int32_t E, int32_t k) {
    const int64_t R = S * k;
    MlpBwdLayout L;
    size_t o = 0;
    L.status = o; o += kStatusBytes;
    L.dhp = o; o = align_up(o + 2 * (size_t)R * (size_t)F);
    // [da | db], the gated dout rows and the router's dl in the weight gradient's padded layout
    const int64_t Rp = R + (int64_t)kWgradPad * E;
    L.dpre = o; o = align_up(o + 4 * (size_t)Rp * (size_t)F);
    L.dw = o; o = align_up(o + 4 * (size_t)R);
    L.dv = o; o = align_up(o + 2 * (size_t)Rp * (size_t)D);
    const int32_t P = router_chunks(S, D);
    L.dl = o; o = align_up(o + 2 * (size_t)(S + (int64_t)kWgradPad * P) * (size_t)E);
    L.xs = o; o = align_up(o + 2 * (size_t)R * (size_t)D);
    L.off1 = o; o = align_up(o + sizeof(int32_t) * (size_t)(P + 1));
    L.partial = o; o = align_up(o + sizeof(float) * (size_t)P * (size_t)D * (size_t)E);
    L.wgt = o; o = align_up(o + 2 * (size_t)E * (size_t)D);
    L.total = o;
    return L;
}

size_t map_ws_bytes(int64_t S, int32_t E, int32_t k) {
    return kStatusBytes + align_up(map_scratch_bytes(S * k, E));
}

int check_ws(void *ws, size_t ws_bytes, size_t need) {
    if (ws == nullptr) return set_error(MOE_ERR_WORKSPACE, "workspace is null");
    if (!aligned(ws, kAlign)) return set_error(MOE_ERR_WORKSPACE, "workspace is not 256-byte aligned");
    if (ws_bytes < need)
        return set_error(MOE_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", ws_bytes, need);
    return MOE_OK;
}

template <class T>
T *at(void *ws, size_t off) {
    return reinterpret_cast<T *>(static_cast<uint8_t *>(ws) + off);
}

void record_prof(int idx, cudaStream_t s) {
    if (g_prof_n > idx && g_prof_events[idx] != nullptr)
        cudaEventRecord(static_cast<cudaEvent_t>(g_prof_events[idx]), s);
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

const char *moe_last_error(void) { return g_err; }

int moe_last_launch_count(void) { return g_launches; }

int moe_profile_events(void *const *events, int n) {
    if (n < 0 || n > 8 || (n > 0 && events == nullptr))
        return set_error(MOE_ERR_INVALID_ARG, "profile events: n must be in [0, 8]");
    g_prof_n = n;
    for (int i = 0; i < n; ++i) g_prof_events[i] = events[i];
    return MOE_OK;
}

size_t moe_workspace_size(const char *op, int64_t S, int64_t D, int64_t F, int32_t E, int32_t k,
                          moe_dtype dt) {
    (void)D;
    if (op == nullptr || S < 0 || E < 1 || E > 256 || k < 1 || k > 8 || k > E) return 0;
    if (S * (int64_t)k >= (int64_t(1) << 31)) return 0;
    if (strcmp(op, "sparse_map") == 0) return map_ws_bytes(S, E, k);
    if (strcmp(op, "scatter_linear") == 0) return kStatusBytes;
    if (strcmp(op, "scatter_linear_backward") == 0) {
        if (F <= 0) return 0;
        if (D <= 0) return 0;
        return bwd_layout(S, D, F, E, k).total;  // D = Din, F = Dout
    }
    if (strcmp(op, "mlp_backward") == 0) {
        if (F <= 0 || D <= 0) return 0;
        return mlp_bwd_layout(S, D, F, E, k).total;
    }
    if (strcmp(op, "moa_forward") == 0) {  // F = H * dh
        if (F <= 0 || dt != MOE_BF16) return 0;
        return moa_layout(S, F, E, k).total;
    }
    if (strcmp(op, "ep_dispatch") == 0) return map_ws_bytes(S, E, k);
    if (strcmp(op, "expert_mlp_forward") == 0) {  // S = rows, k = 1
        if (F <= 0 || k != 1 || (dt != MOE_F32 && dt != MOE_BF16)) return 0;
        return mlp_layout(S, D, F, E, 1, dt, false).total;
    }
    if (strcmp(op, "mlp_forward") == 0) {
        if (F <= 0 || (dt != MOE_F32 && dt != MOE_BF16)) return 0;
        return mlp_layout(S, D, F, E, k, dt).total;
    }
    return 0;
}

int64_t moe_workspace_view(const char *which, int64_t S, int64_t D, int64_t F, int32_t E,
                           int32_t k, moe_dtype dt) {
    if (which == nullptr) return -1;
    const MlpLayout L = mlp_layout(S, D, F, E, k, dt);
    if (!strcmp(which, "top_experts")) return (int64_t)L.top_e;
    if (!strcmp(which, "top_weights")) return (int64_t)L.top_w;
    if (!strcmp(which, "expert_counts")) return (int64_t)L.counts;
    if (!strcmp(which, "expert_offsets")) return (int64_t)L.offsets;
    if (!strcmp(which, "sparse_rows")) return (int64_t)L.sparse_rows;
    if (!strcmp(which, "sorted_rows")) return (int64_t)L.sorted_rows;
    if (!strcmp(which, "h")) return (int64_t)L.h;
    if (!strcmp(which, "x_sorted")) return L.xs_bytes > 0 ? (int64_t)L.xs : -1;
    return -1;
}

int moe_route_topk(const void *x, const void *w_gate, const float *logit_bias, int64_t S,
                   int64_t D, int32_t E, int32_t k, moe_dtype dt, int32_t *top_experts,
                   float *top_weights, moe_stream_t stream) {
    g_launches = 0;
    int rc;
    if ((rc = check_dtype(dt)) || (rc = check_dims(S, E, k)) || (rc = check_feat("D", D))) return rc;
    const size_t eb = esize(dt);
    (void)eb;
    if ((rc = check_ptr("x", x, 16)) || (rc = check_ptr("w_gate", w_gate, 16)) ||
        (rc = check_ptr("logit_bias", logit_bias, 4, true)) ||
        (rc = check_ptr("top_experts", top_experts, 4)) ||
        (rc = check_ptr("top_weights", top_weights, 4)))
        return rc;
    if ((rc = check_device())) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // no workspace in this call: a device-side wait timeout of the tensor-core router is not
    // reported here (moe_mlp_forward reports it through its workspace)
    const int n = launch_route(x, w_gate, logit_bias, S, D, E, k, dt == MOE_BF16, top_experts,
                               top_weights, nullptr, s);
    if (n < 0) return MOE_ERR_CUDA;
    g_launches = n;
    return check_launch("route");
}

int moe_sparse_map(const int32_t *top_experts, int64_t S, int32_t k, int32_t E,
                   int32_t *expert_counts, int32_t *expert_offsets, int32_t *sparse_rows,
                   int32_t *sorted_rows, void *ws, size_t ws_bytes, moe_stream_t stream) {
    g_launches = 0;
    int rc;
    if ((rc = check_dims(S, E, k))) return rc;
    const int64_t R = S * k;
    if ((rc = check_ptr("top_experts", top_experts, 4, R == 0)) ||
        (rc = check_ptr("expert_counts", expert_counts, 4)) ||
        (rc = check_ptr("expert_offsets", expert_offsets, 4)) ||
        (rc = check_ptr("sparse_rows", sparse_rows, 4, R == 0)) ||
        (rc = check_ptr("sorted_rows", sorted_rows, 4, R == 0)))
        return rc;
    if ((rc = check_ws(ws, ws_bytes, map_ws_bytes(S, E, k)))) return rc;
    if ((rc = check_device())) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    unsigned *status = at<unsigned>(ws, 0);
    if (cudaMemsetAsync(status, 0, sizeof(unsigned), s) != cudaSuccess)
        return set_error(MOE_ERR_CUDA, "cudaMemsetAsync of the status word failed");
    int n = 0;
    launch_sparse_map(top_experts, R, E, expert_counts, expert_offsets, sparse_rows, sorted_rows,
                      at<int32_t>(ws, kStatusBytes), status, s, &n);
    g_launches = n;
    return check_launch("sparse_map");
}

int moe_scatter_linear(const void *X, const void *W, int64_t S, int64_t Din, int64_t Dout,
                       int32_t E, int32_t k, const int32_t *sorted_rows,
                       const int32_t *expert_offsets, const float *top_weights, int gather_in,
                       int scatter_out, moe_dtype dt, void *Y, void *ws, size_t ws_bytes,
                       moe_stream_t stream) {
    g_launches = 0;
    int rc;
    if ((rc = check_dtype(dt)) || (rc = check_dims(S, E, k)) || (rc = check_feat("Din", Din)) ||
        (rc = check_feat("Dout", Dout)))
        return rc;
    const int64_t R = S * k;
    if ((rc = check_ptr("X", X, 16, R == 0)) || (rc = check_ptr("W", W, 16)) ||
        (rc = check_ptr("sorted_rows", sorted_rows, 4, R == 0)) ||
        (rc = check_ptr("expert_offsets", expert_offsets, 4)) ||
        (rc = check_ptr("top_weights", top_weights, 4, true)) || (rc = check_ptr("Y", Y, 16, R == 0)))
        return rc;
    if ((rc = check_ws(ws, ws_bytes, kStatusBytes))) return rc;
    if ((rc = check_device())) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    unsigned *status = at<unsigned>(ws, 0);
    if (cudaMemsetAsync(status, 0, sizeof(unsigned), s) != cudaSuccess)
        return set_error(MOE_ERR_CUDA, "cudaMemsetAsync of the status word failed");
    if (R == 0) return MOE_OK;
    GemmArgs a{};
    a.A = X;
    a.a_rows = gather_in ? S : R;
    a.B0 = W;
    a.B1 = nullptr;
    a.offsets = expert_offsets;
    a.sorted_rows = sorted_rows;
    a.gates = top_weights;
    a.out = Y;
    a.S = S;
    a.R = R;
    a.E = E;
    a.k = k;
    a.K = Din;
    a.N = Dout;
    a.bf16 = dt == MOE_BF16;
    a.gather = gather_in != 0;
    a.glu = false;
    a.scatter = scatter_out != 0;
    a.status = status;
    a.wait_limit_ns = kWaitLimitNs;
    if ((rc = prefer_2sm(R, E) ? launch_grouped_gemm_2sm(a, s) : launch_grouped_gemm(a, s)))
        return rc;
    g_launches = 1;
    return check_launch("scatter_linear");
}

int moe_scatter_linear_backward(const void *X, const void *W, const void *dY, int64_t S,
                                int64_t Din, int64_t Dout, int32_t E, int32_t k,
                                const int32_t *sorted_rows, const int32_t *expert_offsets,
                                const float *top_weights, int gather_in, int scatter_out,
                                moe_dtype dt, void *dX, float *dW, float *dgates, void *ws,
                                size_t ws_bytes, moe_stream_t stream) {
    g_launches = 0;
    int rc;
    if ((rc = check_dtype(dt)) || (rc = check_dims(S, E, k)) || (rc = check_feat("Din", Din)) ||
        (rc = check_feat("Dout", Dout)))
        return rc;
    if (dt != MOE_BF16)
        return set_error(MOE_ERR_UNSUPPORTED, "scatter_linear_backward: bf16 inputs only");
    if (dgates != nullptr && top_weights == nullptr)
        return set_error(MOE_ERR_INVALID_ARG, "dgates needs top_weights (the forward's gates)");
    const int64_t R = S * k;
    if ((rc = check_ptr("X", X, 16, R == 0)) || (rc = check_ptr("W", W, 16)) ||
        (rc = check_ptr("dY", dY, 16, R == 0)) ||
        (rc = check_ptr("sorted_rows", sorted_rows, 4, R == 0)) ||
        (rc = check_ptr("expert_offsets", expert_offsets, 4)) ||
        (rc = check_ptr("top_weights", top_weights, 4, true)) ||
        (rc = check_ptr("dX", dX, 16, true)) || (rc = check_ptr("dW", dW, 16, true)) ||
        (rc = check_ptr("dgates", dgates, 16, true)))
        return rc;
    const BwdLayout L = bwd_layout(S, Din, Dout, E, k);
    if ((rc = check_ws(ws, ws_bytes, L.total))) return rc;
    if ((rc = check_device())) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    unsigned *status = at<unsigned>(ws, L.status);
    if (cudaMemsetAsync(status, 0, sizeof(unsigned), s) != cudaSuccess)
        return set_error(MOE_ERR_CUDA, "cudaMemsetAsync of the status word failed");
    int n = 0;
    // input gradient accumulates into token rows: start from zero
    if (dX != nullptr && gather_in) {
        launch_zero_f32(static_cast<float *>(dX), S * Din, nullptr, s);
        ++n;
    }
    if (R == 0) {
        if (dW != nullptr) {
            launch_zero_f32(dW, (int64_t)E * Din * Dout, nullptr, s);
            ++n;
        }
        g_launches = n;
        return check_launch("scatter_linear_backward");
    }
    // the output gradient as a bf16 operand: dY is fp32 [S, Dout] when the forward scattered
    const void *dyb = dY;
    if (scatter_out) {
        launch_cast_bf16(static_cast<const float *>(dY), at<void>(ws, L.dyb), S * Dout, s);
        dyb = at<void>(ws, L.dyb);
        ++n;
    }
    GemmArgs a{};
    a.offsets = expert_offsets;
    a.sorted_rows = sorted_rows;
    a.S = S;
    a.R = R;
    a.E = E;
    a.k = k;
    a.bf16 = true;
    a.glu = false;
    a.status = status;
    a.wait_limit_ns = kWaitLimitNs;
    if (dX != nullptr) {
        // dX = ParallelLinear(dY, W^T, I, G) with the gather and scatter roles exchanged
        GemmArgs b = a;
        b.A = dyb;
        b.a_rows = scatter_out ? S : R;
        b.B0 = W;  // [E, Din, Dout] read K-major as W^T: N = Din, K = Dout
        b.b_kmajor = true;
        b.gates = top_weights;
        b.out = dX;
        b.K = Dout;
        b.N = Din;
        b.gather = scatter_out != 0;
        b.scatter = gather_in != 0;
        if ((rc = launch_grouped_gemm(b, s))) return rc;
        ++n;
    }
    if (dW != nullptr) {
        // B: the gated dY rows in the padded layout; A: the input rows in slot order
        launch_gate_rows(dY, !scatter_out, sorted_rows, top_weights, k, R, Dout, scatter_out != 0,
                         at<void>(ws, L.dv), expert_offsets, E, status, s);
        launch_zero_pad_rows(at<void>(ws, L.dv), Dout, Dout, expert_offsets, E, s);
        const void *As = X;
        if (gather_in) {
            launch_gather_rows(X, sorted_rows, k, R, Din, at<void>(ws, L.xs), status, s);
            As = at<void>(ws, L.xs);
            ++n;
        }
        WgradArgs w{};
        w.A = As;
        w.a_rows = R;
        w.dv = at<void>(ws, L.dv);
        w.dv_rows = R + (int64_t)kWgradPad * E;
        w.offsets = expert_offsets;
        w.Din = Din;
        w.Dout = Dout;
        w.E = E;
        w.dW = dW;
        w.status = status;
        w.wait_limit_ns = kWaitLimitNs;
        if ((rc = launch_grouped_wgrad(w, s))) return rc;
        n += 3;
    }
    if (dgates != nullptr) {
        // v = the ungated forward rows in slot order; dgates[i] = dY[row] . v[p]
        GemmArgs f = a;
        f.A = X;
        f.a_rows = gather_in ? S : R;
        f.B0 = W;
        f.gates = nullptr;
        f.out = at<void>(ws, L.v);
        f.K = Din;
        f.N = Dout;
        f.gather = gather_in != 0;
        f.scatter = false;
        if ((rc = prefer_2sm(R, E) ? launch_grouped_gemm_2sm(f, s) : launch_grouped_gemm(f, s)))
            return rc;
        launch_zero_f32(dgates, R, nullptr, s);
        launch_rowdot(dY, !scatter_out, at<void>(ws, L.v), sorted_rows, k, R, Dout,
                      scatter_out != 0, dgates, status, s);
        n += 3;
    }
    g_launches = n;
    return check_launch("scatter_linear_backward");
}

int moe_mlp_forward(const void *x, const void *w_gate, const float *logit_bias,
                    const void *w_gate_e, const void *w_up, const void *w_down, int64_t S,
                    int64_t D, int64_t F, int32_t E, int32_t k, moe_dtype dt, float *out, void *ws,
                    size_t ws_bytes, moe_stream_t stream) {
    g_launches = 0;
    int rc;
    if ((rc = check_dtype(dt)) || (rc = check_dims(S, E, k)) || (rc = check_feat("D", D)) ||
        (rc = check_feat("F", F)))
        return rc;
    if ((rc = check_ptr("x", x, 16, S == 0)) || (rc = check_ptr("w_gate", w_gate, 16)) ||
        (rc = check_ptr("logit_bias", logit_bias, 4, true)) ||
        (rc = check_ptr("w_gate_e", w_gate_e, 16)) || (rc = check_ptr("w_up", w_up, 16)) ||
        (rc = check_ptr("w_down", w_down, 16)) || (rc = check_ptr("out", out, 16, S == 0)))
        return rc;
    const MlpLayout L = mlp_layout(S, D, F, E, k, dt);
    if ((rc = check_ws(ws, ws_bytes, L.total))) return rc;
    if ((rc = check_device())) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int64_t R = S * k;
    unsigned *status = at<unsigned>(ws, L.status);
    int32_t *top_e = at<int32_t>(ws, L.top_e);
    float *top_w = at<float>(ws, L.top_w);
    int32_t *counts = at<int32_t>(ws, L.counts);
    int32_t *offsets = at<int32_t>(ws, L.offsets);
    int32_t *sparse_rows = at<int32_t>(ws, L.sparse_rows);
    int32_t *sorted_rows = at<int32_t>(ws, L.sorted_rows);
    void *h = at<void>(ws, L.h);
    int n = 0;

    record_prof(0, s);
    // The router clears the status word (its first kernel); GEMM1's epilogue warps zero `out`
    // while they wait for their first tile. With no routes there is no GEMM: a small kernel does
    // both.
    if (R == 0) {
        n += launch_zero_f32(out, S * D, status, s);
        if ((rc = check_launch("zero"))) return rc;
    }
    {
        const int nr = launch_route(x, w_gate, logit_bias, S, D, E, k, dt == MOE_BF16, top_e,
                                    top_w, status, s);
        if (nr < 0) return MOE_ERR_CUDA;
        n += nr;
    }
    if ((rc = check_launch("route"))) return rc;
    record_prof(1, s);
    launch_sparse_map(top_e, R, E, counts, offsets, sparse_rows, sorted_rows,
                      at<int32_t>(ws, L.scratch), status, s, &n);
    if ((rc = check_launch("sparse_map"))) return rc;
    record_prof(2, s);
    if (R > 0) {
        // x rows copied to slot order first (the gather's own kernel), so that GEMM1 loads them
        // by TMA like GEMM2's h rows; otherwise GEMM1 gathers them on load
        const bool pregather = L.xs_bytes > 0 && !env_off("MOE_PREGATHER");
        void *xs = at<void>(ws, L.xs);
        if (pregather) {
            launch_gather_rows(x, sorted_rows, k, R, D, xs, status, s);
            if ((rc = check_launch("gather_rows"))) return rc;
            ++n;
        }
        record_prof(3, s);
        GemmArgs a{};
        a.A = pregather ? xs : x;
        a.a_rows = pregather ? R : S;
        a.B0 = w_gate_e;
        a.B1 = w_up;
        a.offsets = offsets;
        a.sorted_rows = sorted_rows;
        a.gates = nullptr;
        a.out = h;
        a.S = S;
        a.R = R;
        a.E = E;
        a.k = k;
        a.K = D;
        a.N = F;
        a.bf16 = dt == MOE_BF16;
        a.gather = !pregather;
        a.glu = true;
        a.scatter = false;
        a.zero_ptr = out;   // zeroed by GEMM1's epilogue warps before GEMM2 adds into it
        a.zero_n = S * D;
        a.status = status;
        a.wait_limit_ns = kWaitLimitNs;
        if ((rc = prefer_2sm(R, E) ? launch_grouped_gemm_2sm(a, s) : launch_grouped_gemm(a, s)))
            return rc;
        if ((rc = check_launch("gemm1"))) return rc;
        ++n;
        record_prof(4, s);
        GemmArgs b = a;
        b.zero_ptr = nullptr;
        b.zero_n = 0;
        b.A = h;
        b.a_rows = R;
        b.B0 = w_down;
        b.B1 = nullptr;
        b.gates = top_w;
        b.out = out;
        b.K = F;
        b.N = D;
        b.gather = false;
        b.glu = false;
        b.scatter = true;
        if ((rc = prefer_2sm_scatter(R, E) ? launch_grouped_gemm_2sm(b, s) : launch_grouped_gemm(b, s)))
            return rc;
        if ((rc = check_launch("gemm2"))) return rc;
        ++n;
        record_prof(5, s);
    } else {
        record_prof(3, s);
        record_prof(4, s);
        record_prof(5, s);
    }
    g_prof_n = 0;
    g_launches = n;
    return MOE_OK;
}

int moe_check_device_status(void *ws, moe_stream_t stream) {
    if (ws == nullptr) return set_error(MOE_ERR_WORKSPACE, "workspace is null");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return set_error(MOE_ERR_CUDA, "stream: %s", cudaGetErrorString(e));
    unsigned v = 0;
    e = cudaMemcpy(&v, ws, sizeof(v), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return set_error(MOE_ERR_CUDA, "status read: %s", cudaGetErrorString(e));
    if (v & kStatusTimeout)
        return set_error(MOE_ERR_DEVICE_TIMEOUT, "a device wait ran out (kernel id %u)", (v >> 8) & 0xFFu);
    if (v & kStatusBadExpert)
        return set_error(MOE_ERR_BAD_EXPERT_ID, "an expert id outside [0, E) was seen");
    if (v & kStatusBadIndex)
        return set_error(MOE_ERR_BAD_INDEX,
                         "a device bounds check skipped an index outside its range");
    return MOE_OK;
}

int moe_debug_build(void) { return kDebugChecks ? 1 : 0; }

int moe_debug_wait_timeout(int64_t limit_ns, void *ws, size_t ws_bytes, moe_stream_t stream) {
    g_launches = 0;
    int rc;
    if (limit_ns < 1 || limit_ns > 1000000000LL)
        return set_error(MOE_ERR_INVALID_ARG, "limit_ns must be in [1, 1e9]");
    if ((rc = check_ws(ws, ws_bytes, kStatusBytes))) return rc;
    if ((rc = check_device())) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    unsigned *status = at<unsigned>(ws, 0);
    if (cudaMemsetAsync(status, 0, sizeof(unsigned), s) != cudaSuccess)
        return set_error(MOE_ERR_CUDA, "cudaMemsetAsync of the status word failed");
    launch_debug_wait(limit_ns, status, s);
    g_launches = 1;
    return check_launch("debug_wait");
}

}  // extern "C"

extern "C" int moe_mlp_backward(const void *x, const void *w_gate, const void *w_gate_e,
                                const void *w_up, const void *w_down, const float *dout, int64_t S,
                                int64_t D, int64_t F, int32_t E, int32_t k, moe_dtype dt,
                                const void *fwd_ws, size_t fwd_ws_bytes, float *dx, float *dw_gate,
                                float *dw_gate_e, float *dw_up, float *dw_down, void *ws,
                                size_t ws_bytes, moe_stream_t stream) {
    g_launches = 0;
    int rc;
    if ((rc = check_dtype(dt)) || (rc = check_dims(S, E, k)) || (rc = check_feat("D", D)) ||
        (rc = check_feat("F", F)))
        return rc;
    if (dt != MOE_BF16) return set_error(MOE_ERR_UNSUPPORTED, "mlp_backward: bf16 inputs only");
    if (E % 8 != 0)
        return set_error(MOE_ERR_UNSUPPORTED, "mlp_backward: E must be a multiple of 8 (got %d)", E);
    if (F % 64 != 0)
        return set_error(MOE_ERR_UNSUPPORTED, "mlp_backward: F must be a multiple of 64 (got %lld)",
                         (long long)F);
    const int64_t R = S * k;
    if ((rc = check_ptr("x", x, 16, S == 0)) || (rc = check_ptr("w_gate", w_gate, 16)) ||
        (rc = check_ptr("w_gate_e", w_gate_e, 16)) || (rc = check_ptr("w_up", w_up, 16)) ||
        (rc = check_ptr("w_down", w_down, 16)) || (rc = check_ptr("dout", dout, 16, S == 0)) ||
        (rc = check_ptr("dx", dx, 16, S == 0)) || (rc = check_ptr("dw_gate", dw_gate, 16)) ||
        (rc = check_ptr("dw_gate_e", dw_gate_e, 16)) || (rc = check_ptr("dw_up", dw_up, 16)) ||
        (rc = check_ptr("dw_down", dw_down, 16)))
        return rc;
    const MlpLayout FL = mlp_layout(S, D, F, E, k, dt);
    if (fwd_ws == nullptr || fwd_ws_bytes < FL.total)
        return set_error(MOE_ERR_WORKSPACE, "the forward's workspace is missing or too small");
    const MlpBwdLayout L = mlp_bwd_layout(S, D, F, E, k);
    if ((rc = check_ws(ws, ws_bytes, L.total))) return rc;
    if ((rc = check_device())) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    void *fws = const_cast<void *>(fwd_ws);
    const int32_t *top_e = at<int32_t>(fws, FL.top_e);
    const float *top_w = at<float>(fws, FL.top_w);
    const int32_t *offsets = at<int32_t>(fws, FL.offsets);
    const int32_t *sorted_rows = at<int32_t>(fws, FL.sorted_rows);
    const void *h = at<void>(fws, FL.h);
    unsigned *status = at<unsigned>(ws, L.status);
    if (cudaMemsetAsync(status, 0, sizeof(unsigned), s) != cudaSuccess)
        return set_error(MOE_ERR_CUDA, "cudaMemsetAsync of the status word failed");
    int n = 0;
    launch_zero_f32(dx, S * D, nullptr, s);
    ++n;
    if (R == 0) {
        launch_zero_f32(dw_gate, D * E, nullptr, s);
        launch_zero_f32(dw_gate_e, (int64_t)E * D * F, nullptr, s);
        launch_zero_f32(dw_up, (int64_t)E * D * F, nullptr, s);
        launch_zero_f32(dw_down, (int64_t)E * F * D, nullptr, s);
        g_launches = n + 4;
        return check_launch("mlp_backward");
    }
    // profile events (moe_profile_events): 0 start, 1 after dh, 2 after the GEMM1 recompute with
    // the SwiGLU backward, 3 after dW_down, 4 after dx, 5 after dW_gate_e/dW_up, 6 end
    record_prof(0, s);
    void *dhp = at<void>(ws, L.dhp);
    void *dpre = at<void>(ws, L.dpre), *dv = at<void>(ws, L.dv);
    void *dl = at<void>(ws, L.dl);
    float *dwr = at<float>(ws, L.dw);
    int32_t *off1 = at<int32_t>(ws, L.off1);
    // dout rows (bf16, ungated) in slot order, in the padded layout of dv (the weight gradient
    // refills dv with the gated rows below); dh then reads them by TMA instead of gathering them
    launch_gate_rows(dout, false, sorted_rows, nullptr, k, R, D, true, dv, offsets, E, status, s);
    ++n;
    // x rows in slot order: read by TMA in the GEMM1 recompute, then by the W_gate_e / W_up
    // weight gradient
    void *xs = at<void>(ws, L.xs);
    launch_gather_rows(x, sorted_rows, k, R, D, xs, status, s);
    ++n;
    const int64_t Rp = R + (int64_t)kWgradPad * E;
    GemmArgs g{};
    g.offsets = offsets;
    g.sorted_rows = sorted_rows;
    g.S = S;
    g.R = R;
    g.E = E;
    g.k = k;
    g.bf16 = true;
    g.status = status;
    g.wait_limit_ns = kWaitLimitNs;
    // GEMM2 backward, ungated: dhp[p] = dout[s] . W_down[e]^T (W_down [E, F, D] read K-major)
    {
        GemmArgs a = g;
        a.A = dv;
        a.a_rows = Rp;
        a.a_row_pad = kWgradPad;
        a.B0 = w_down;
        a.b_kmajor = true;
        a.out = dhp;
        a.K = D;
        a.N = F;
        a.gather = false;
        if ((rc = prefer_2sm(R, E) ? launch_grouped_gemm_2sm(a, s) : launch_grouped_gemm(a, s)))
            return rc;
        ++n;
    }
    record_prof(1, s);
    // GEMM1 recomputed (fused gate+up, slot-ordered x) with the SwiGLU backward in its epilogue: the
    // route-weight gradient dh_u . h (atomically per N tile) and [da | db] in the padded layout
    launch_zero_f32(dwr, R, nullptr, s);
    {
        GemmArgs a = g;
        a.A = xs;
        a.a_rows = R;
        a.B0 = w_gate_e;
        a.B1 = w_up;
        a.gates = top_w;
        a.out = dpre;
        a.K = D;
        a.N = F;
        a.gather = false;
        a.glu = true;
        a.glu_bwd = true;
        a.bwd_dh = dhp;
        a.bwd_dw = dwr;
        a.out_row_pad = kWgradPad;
        if ((rc = prefer_2sm(R, E) ? launch_grouped_gemm_2sm(a, s) : launch_grouped_gemm(a, s)))
            return rc;
    }
    launch_zero_pad_rows(dpre, 2 * F, 2 * F, offsets, E, s);
    n += 3;
    record_prof(2, s);
    // dW_down[e] = sum over e's slots of h_p^T (w_i dout[s])
    launch_gate_rows(dout, false, sorted_rows, top_w, k, R, D, true, dv, offsets, E, status, s);
    launch_zero_pad_rows(dv, D, D, offsets, E, s);
    {
        WgradArgs w{};
        w.A = h;
        w.a_rows = R;
        w.dv = dv;
        w.dv_rows = Rp;
        w.offsets = offsets;
        w.Din = F;
        w.Dout = D;
        w.E = E;
        w.dW = dw_down;
        w.status = status;
        w.wait_limit_ns = kWaitLimitNs;
        if ((rc = launch_grouped_wgrad(w, s))) return rc;
        n += 3;
    }
    record_prof(3, s);
    // dx (experts) += [da | db] . [W_gate_e ; W_up]^T, scatter-added into tokens
    {
        GemmArgs a = g;
        a.A = dpre;
        a.a_rows = Rp;
        a.a_row_pad = kWgradPad;
        a.B0 = w_gate_e;
        a.B1 = w_up;
        a.k_split = F;
        a.b_kmajor = true;
        a.out = dx;
        a.K = 2 * F;
        a.N = D;
        a.gather = false;
        a.scatter = true;
        if ((rc = prefer_2sm(R, E) ? launch_grouped_gemm_2sm(a, s) : launch_grouped_gemm(a, s)))
            return rc;
        ++n;
    }
    record_prof(4, s);
    // dW_gate_e, dW_up from the x rows in slot order and the two halves of [da | db]
    for (int half = 0; half < 2; ++half) {
        WgradArgs w{};
        w.A = xs;
        w.a_rows = R;
        w.dv = static_cast<const uint8_t *>(dpre) + (size_t)half * F * 2;
        w.dv_rows = Rp;
        w.dv_ld = 2 * F;
        w.offsets = offsets;
        w.Din = D;
        w.Dout = F;
        w.E = E;
        w.dW = half == 0 ? dw_gate_e : dw_up;
        w.status = status;
        w.wait_limit_ns = kWaitLimitNs;
        if ((rc = launch_grouped_wgrad(w, s))) return rc;
        ++n;
    }
    record_prof(5, s);
    // router: dl (softmax over the selection), dx += dl W_gate^T, dW_gate = x^T dl
    // the W_gate gradient in P token chunks (partial gradients), then summed
    const int32_t P = router_chunks(S, D);
    const int32_t chunk = (int32_t)((S + P - 1) / P);
    float *partial = at<float>(ws, L.partial);
    launch_router_bwd(top_e, top_w, dwr, w_gate, at<void>(ws, L.wgt), S, D, E, k, dl, dx, off1,
                      chunk, P, s);
    launch_zero_pad_rows(dl, E, E, off1, P, s);
    n += 3;
    {
        WgradArgs w{};
        w.A = x;
        w.a_rows = S;
        w.dv = dl;
        w.dv_rows = S + (int64_t)kWgradPad * P;
        w.offsets = off1;
        w.Din = D;
        w.Dout = E;
        w.E = P;
        w.dW = partial;
        w.status = status;
        w.wait_limit_ns = kWaitLimitNs;
        if ((rc = launch_grouped_wgrad(w, s))) return rc;
        launch_sum_partials(partial, D * E, P, dw_gate, s);
        n += 2;
    }
    record_prof(6, s);
    g_prof_n = 0;
    g_launches = n;
    return check_launch("mlp_backward");
}

int moe_moa_forward(const void *x, const void *w_gate, const float *logit_bias, const void *w_q,
                    const void *w_kv, const void *w_o, int64_t S, int64_t D, int32_t H, int32_t dh,
                    int32_t E, int32_t k, moe_dtype dt, float *out, void *ws, size_t ws_bytes,
                    moe_stream_t stream) {
    g_launches = 0;
    int rc;
    if ((rc = check_dtype(dt)) || (rc = check_dims(S, E, k)) || (rc = check_feat("D", D)))
        return rc;
    if (dt != MOE_BF16) return set_error(MOE_ERR_UNSUPPORTED, "moa_forward: bf16 inputs only");
    if (dh != 64 && dh != 128)
        return set_error(MOE_ERR_UNSUPPORTED, "moa_forward: head size %d (64 or 128 are built)", dh);
    if (H < 1 || (int64_t)H * dh * 2 >= (int64_t(1) << 31))
        return set_error(MOE_ERR_INVALID_ARG, "moa_forward: H must be positive with 2*H*dh < 2^31");
    const int64_t HD = (int64_t)H * dh;
    if ((rc = check_ptr("x", x, 16, S == 0)) || (rc = check_ptr("w_gate", w_gate, 16)) ||
        (rc = check_ptr("logit_bias", logit_bias, 4, true)) || (rc = check_ptr("w_q", w_q, 16)) ||
        (rc = check_ptr("w_kv", w_kv, 16)) || (rc = check_ptr("w_o", w_o, 16)) ||
        (rc = check_ptr("out", out, 16, S == 0)))
        return rc;
    const MoaLayout L = moa_layout(S, HD, E, k);
    if ((rc = check_ws(ws, ws_bytes, L.total))) return rc;
    if ((rc = check_device())) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int64_t R = S * k;
    unsigned *status = at<unsigned>(ws, L.base.status);
    int32_t *top_e = at<int32_t>(ws, L.base.top_e);
    float *top_w = at<float>(ws, L.base.top_w);
    int32_t *offsets = at<int32_t>(ws, L.base.offsets);
    int32_t *sorted_rows = at<int32_t>(ws, L.base.sorted_rows);
    int32_t *kv_off = at<int32_t>(ws, L.kv_off);
    void *kv = at<void>(ws, L.kv), *q = at<void>(ws, L.q), *o = at<void>(ws, L.o);
    int n = 0;

    record_prof(0, s);
    if (R == 0) {
        n += launch_zero_f32(out, S * D, status, s);
        if ((rc = check_launch("zero"))) return rc;
    }
    {
        const int nr = launch_route(x, w_gate, logit_bias, S, D, E, k, true, top_e, top_w, status, s);
        if (nr < 0) return MOE_ERR_CUDA;
        n += nr;
    }
    if ((rc = check_launch("route"))) return rc;
    record_prof(1, s);
    launch_sparse_map(top_e, R, E, at<int32_t>(ws, L.base.counts), offsets,
                      at<int32_t>(ws, L.base.sparse_rows), sorted_rows,
                      at<int32_t>(ws, L.base.scratch), status, s, &n);
    if ((rc = check_launch("sparse_map"))) return rc;
    record_prof(2, s);
    if (R > 0) {
        // shared keys and values: one group of all S tokens, [S, D] . [D, 2 HD]; its epilogue
        // warps also zero `out` for the final scatter-add
        launch_kv_offsets(kv_off, S, s);
        GemmArgs a{};
        a.A = x;
        a.a_rows = S;
        a.B0 = w_kv;
        a.offsets = kv_off;
        a.sorted_rows = sorted_rows;
        a.out = kv;
        a.S = S;
        a.R = S;
        a.E = 1;
        a.k = 1;
        a.K = D;
        a.N = 2 * HD;
        a.bf16 = true;
        a.zero_ptr = out;
        a.zero_n = S * D;
        a.status = status;
        a.wait_limit_ns = kWaitLimitNs;
        if ((rc = prefer_2sm(S, 1) ? launch_grouped_gemm_2sm(a, s) : launch_grouped_gemm(a, s)))
            return rc;
        if ((rc = check_launch("kv projection"))) return rc;
        n += 2;
        record_prof(3, s);
        // routed query projection: gathered x rows, W_q[e], q in slot order
        GemmArgs b{};
        b.A = x;
        b.a_rows = S;
        b.B0 = w_q;
        b.offsets = offsets;
        b.sorted_rows = sorted_rows;
        b.out = q;
        b.S = S;
        b.R = R;
        b.E = E;
        b.k = k;
        b.K = D;
        b.N = HD;
        b.bf16 = true;
        b.gather = true;
        b.status = status;
        b.wait_limit_ns = kWaitLimitNs;
        if ((rc = prefer_2sm(R, E) ? launch_grouped_gemm_2sm(b, s) : launch_grouped_gemm(b, s)))
            return rc;
        if ((rc = check_launch("q projection"))) return rc;
        ++n;
        record_prof(4, s);
        if ((rc = launch_moa_attention(q, kv, at<int32_t>(ws, L.base.sparse_rows), o, R, S, H, dh,
                                       k, status, s)))
            return rc;
        if ((rc = check_launch("attention"))) return rc;
        ++n;
        record_prof(5, s);
        // routed output projection: o rows in slot order, W_o[e], router weight, scatter-add
        GemmArgs c = b;
        c.A = o;
        c.a_rows = R;
        c.B0 = w_o;
        c.gates = top_w;
        c.out = out;
        c.K = HD;
        c.N = D;
        c.gather = false;
        c.scatter = true;
        if ((rc = prefer_2sm_scatter(R, E) ? launch_grouped_gemm_2sm(c, s) : launch_grouped_gemm(c, s)))
            return rc;
        if ((rc = check_launch("o projection"))) return rc;
        ++n;
        record_prof(6, s);
    } else {
        for (int q = 3; q <= 6; ++q) record_prof(q, s);
    }
    g_prof_n = 0;
    g_launches = n;
    return MOE_OK;
}

int moe_ep_dispatch(const void *x, const int32_t *top_experts, int64_t S, int64_t D, int32_t E,
                    int32_t k, moe_dtype dt, int32_t *expert_counts, int32_t *expert_offsets,
                    int32_t *sparse_rows, int32_t *sorted_rows, void *send_x, int32_t *send_e,
                    void *ws, size_t ws_bytes, moe_stream_t stream) {
    g_launches = 0;
    int rc;
    if ((rc = check_dtype(dt)) || (rc = check_dims(S, E, k)) || (rc = check_feat("D", D)))
        return rc;
    const int64_t R = S * k;
    if ((rc = check_ptr("x", x, 16, R == 0)) ||
        (rc = check_ptr("top_experts", top_experts, 4, R == 0)) ||
        (rc = check_ptr("expert_counts", expert_counts, 4)) ||
        (rc = check_ptr("expert_offsets", expert_offsets, 4)) ||
        (rc = check_ptr("sparse_rows", sparse_rows, 4, R == 0)) ||
        (rc = check_ptr("sorted_rows", sorted_rows, 4, R == 0)) ||
        (rc = check_ptr("send_x", send_x, 16, R == 0)) ||
        (rc = check_ptr("send_e", send_e, 4, R == 0)))
        return rc;
    if ((rc = check_ws(ws, ws_bytes, map_ws_bytes(S, E, k)))) return rc;
    if ((rc = check_device())) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    unsigned *status = at<unsigned>(ws, 0);
    if (cudaMemsetAsync(status, 0, sizeof(unsigned), s) != cudaSuccess)
        return set_error(MOE_ERR_CUDA, "cudaMemsetAsync of the status word failed");
    int n = 0;
    launch_sparse_map(top_experts, R, E, expert_counts, expert_offsets, sparse_rows, sorted_rows,
                      at<int32_t>(ws, kStatusBytes), status, s, &n);
    if ((rc = check_launch("sparse_map"))) return rc;
    if (R > 0) {
        launch_ep_pack(x, (size_t)D * esize(dt), top_experts, sorted_rows, expert_offsets, E, k,
                       R, send_x, send_e, status, s);
        ++n;
    }
    g_launches = n;
    return check_launch("ep_pack");
}

int moe_expert_mlp_forward(const void *x_rows, const int32_t *expert_ids, int32_t expert_base,
                           int64_t R, int64_t D, int64_t F, int32_t E, const void *w_gate_e,
                           const void *w_up, const void *w_down, moe_dtype dt, float *y, void *ws,
                           size_t ws_bytes, moe_stream_t stream) {
    g_launches = 0;
    int rc;
    if ((rc = check_dtype(dt)) || (rc = check_dims(R, E, 1)) || (rc = check_feat("D", D)) ||
        (rc = check_feat("F", F)))
        return rc;
    if ((rc = check_ptr("x_rows", x_rows, 16, R == 0)) ||
        (rc = check_ptr("expert_ids", expert_ids, 4, R == 0)) ||
        (rc = check_ptr("w_gate_e", w_gate_e, 16)) || (rc = check_ptr("w_up", w_up, 16)) ||
        (rc = check_ptr("w_down", w_down, 16)) || (rc = check_ptr("y", y, 16, R == 0)))
        return rc;
    // the forward's layout with one route per row: top_e holds the local ids
    const MlpLayout L = mlp_layout(R, D, F, E, 1, dt, false);
    if ((rc = check_ws(ws, ws_bytes, L.total))) return rc;
    if ((rc = check_device())) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    unsigned *status = at<unsigned>(ws, L.status);
    int32_t *local = at<int32_t>(ws, L.top_e);
    int32_t *offsets = at<int32_t>(ws, L.offsets);
    int32_t *sorted_rows = at<int32_t>(ws, L.sorted_rows);
    int n = 0;
    launch_local_ids(expert_ids, expert_base, R, local, status, s);
    ++n;
    if ((rc = check_launch("local_ids"))) return rc;
    if (R == 0) {
        g_launches = n;
        return MOE_OK;
    }
    launch_sparse_map(local, R, E, at<int32_t>(ws, L.counts), offsets,
                      at<int32_t>(ws, L.sparse_rows), sorted_rows, at<int32_t>(ws, L.scratch),
                      status, s, &n);
    if ((rc = check_launch("sparse_map"))) return rc;
    GemmArgs a{};
    a.A = x_rows;
    a.a_rows = R;
    a.B0 = w_gate_e;
    a.B1 = w_up;
    a.offsets = offsets;
    a.sorted_rows = sorted_rows;
    a.out = at<void>(ws, L.h);
    a.S = R;
    a.R = R;
    a.E = E;
    a.k = 1;
    a.K = D;
    a.N = F;
    a.bf16 = dt == MOE_BF16;
    a.gather = true;
    a.glu = true;
    a.zero_ptr = y;  // zeroed by GEMM1's epilogue warps before GEMM2 adds into it
    a.zero_n = R * D;
    a.status = status;
    a.wait_limit_ns = kWaitLimitNs;
    if ((rc = prefer_2sm(R, E) ? launch_grouped_gemm_2sm(a, s) : launch_grouped_gemm(a, s)))
        return rc;
    if ((rc = check_launch("gemm1"))) return rc;
    GemmArgs b = a;
    b.zero_ptr = nullptr;
    b.zero_n = 0;
    b.A = at<void>(ws, L.h);
    b.B0 = w_down;
    b.B1 = nullptr;
    b.out = y;
    b.K = F;
    b.N = D;
    b.gather = false;
    b.glu = false;
    b.scatter = true;
    if ((rc = prefer_2sm_scatter(R, E) ? launch_grouped_gemm_2sm(b, s) : launch_grouped_gemm(b, s)))
        return rc;
    n += 2;
    g_launches = n;
    return check_launch("gemm2");
}

int moe_ep_combine(const float *y_ret, const int32_t *sparse_rows, const float *top_weights,
                   int64_t S, int64_t D, int32_t k, float *out, moe_stream_t stream) {
    g_launches = 0;
    int rc;
    if (S < 0 || k < 1 || k > 8 || S * (int64_t)k >= (int64_t(1) << 31))
        return set_error(MOE_ERR_INVALID_ARG, "ep_combine: need S >= 0, 1 <= k <= 8, S*k < 2^31");
    if ((rc = check_feat("D", D))) return rc;
    const int64_t R = S * k;
    if ((rc = check_ptr("y_ret", y_ret, 16, R == 0)) ||
        (rc = check_ptr("sparse_rows", sparse_rows, 4, R == 0)) ||
        (rc = check_ptr("top_weights", top_weights, 4, R == 0)) ||
        (rc = check_ptr("out", out, 16, S == 0)))
        return rc;
    if ((rc = check_device())) return rc;
    if (S == 0) return MOE_OK;
    launch_ep_combine(y_ret, sparse_rows, top_weights, S, k, R, D, out,
                      reinterpret_cast<cudaStream_t>(stream));
    g_launches = 1;
    return check_launch("ep_combine");
}

int moe_cast_bf16(const float *src, int64_t n, void *dst, moe_stream_t stream) {
    g_launches = 0;
    int rc;
    if (n < 0 || n % 8 != 0 || n >= (int64_t(1) << 40))
        return set_error(MOE_ERR_INVALID_ARG, "cast_bf16: n must be a non-negative multiple of 8");
    if ((rc = check_ptr("src", src, 16, n == 0)) || (rc = check_ptr("dst", dst, 16, n == 0)))
        return rc;
    if ((rc = check_device())) return rc;
    if (n == 0) return MOE_OK;
    launch_cast_bf16(src, dst, n, reinterpret_cast<cudaStream_t>(stream));
    g_launches = 1;
    return check_launch("cast_bf16");
}
