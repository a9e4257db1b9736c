// C ABI entry points of libclha.so: argument checks, workspace, dispatch to the kernels, status.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <new>

#include "clha_internal.h"

#define CLHA_VERSION 100

// ------------------------------------------------------------------------------ tracing
#include <atomic>
static std::atomic<int64_t> g_launches{0};
void clha_note_launches(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }
int64_t clha_total_launches() { return g_launches.load(std::memory_order_relaxed); }

extern "C" int64_t clha_kernel_launches(const clha_ctx* ctx) { return ctx ? ctx->launches : 0; }

namespace {
// Adds the kernels launched while it lives to the context's counter.
struct LaunchScope {
    clha_ctx* c;
    int64_t l0;
    explicit LaunchScope(clha_ctx* ctx) : c(ctx), l0(clha_total_launches()) {}
    ~LaunchScope() { c->launches += clha_total_launches() - l0; }
};
}  // namespace

// ------------------------------------------------------------------------------ helpers
clha_status clha_fail(clha_ctx* ctx, clha_status st, const char* fmt, ...) {
    if (ctx) {
        char buf[512];
        va_list ap;
        va_start(ap, fmt);
        vsnprintf(buf, sizeof(buf), fmt, ap);
        va_end(ap);
        ctx->last_error = buf;
    }
    return st;
}

clha_status clha_cuda_check(clha_ctx* ctx, cudaError_t e, const char* what) {
    if (e == cudaSuccess) return CLHA_OK;
    if (e == cudaErrorMemoryAllocation)
        return clha_fail(ctx, CLHA_ERR_OOM, "%s: %s", what, cudaGetErrorString(e));
    return clha_fail(ctx, CLHA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

clha_status clha_launch_check(clha_ctx* ctx, const char* what) {
    return clha_cuda_check(ctx, cudaGetLastError(), what);
}

clha_status clha_workspace(clha_ctx* ctx, size_t bytes, void** out) {
    if (bytes <= ctx->ws_bytes) {
        *out = ctx->ws;
        return CLHA_OK;
    }
    cudaError_t e = cudaStreamSynchronize(ctx->stream);
    if (e != cudaSuccess) return clha_cuda_check(ctx, e, "workspace sync");
    if (ctx->ws) cudaFree(ctx->ws);
    ctx->ws = nullptr;
    ctx->ws_bytes = 0;
    size_t want = bytes + bytes / 8;
    e = cudaMalloc(&ctx->ws, want);
    if (e != cudaSuccess) {
        cudaGetLastError();
        e = cudaMalloc(&ctx->ws, bytes);
        want = bytes;
    }
    if (e != cudaSuccess) {
        cudaGetLastError();
        ctx->ws = nullptr;
        return clha_fail(ctx, CLHA_ERR_OOM, "workspace of %zu bytes: %s", bytes, cudaGetErrorString(e));
    }
    ctx->ws_bytes = want;
    *out = ctx->ws;
    return CLHA_OK;
}

static const char* status_name(int code) {
    switch (code) {
        case CLHA_ERR_NOT_PD: return "non-positive pivot";
        case CLHA_ERR_NONFINITE: return "non-finite value";
        case CLHA_ERR_TIMEOUT: return "device wait timed out";
        case CLHA_ERR_EMPTY: return "no tokens";
        default: return "device error";
    }
}

static const char* kernel_name(int kid) {
    switch (kid) {
        case KID_ROUTE: return "clha_route_topk";
        case KID_GATHER: return "clha_gather";
        case KID_ACT: return "clha_expert_act";
        case KID_COLLECT: return "clha_collect";
        case KID_AGGREGATE: return "clha_aggregate";
        case KID_FACTOR: return "clha_factor";
        case KID_QUANTIZE: return "clha_quantize";
        case KID_LOSS: return "clha_loss";
        case KID_DIVERGENCE: return "clha_routing_divergence";
        default: return "kernel";
    }
}

clha_status clha_sync_and_check(clha_ctx* ctx, const char* call) {
    cudaError_t e = cudaStreamSynchronize(ctx->stream);
    if (e != cudaSuccess) return clha_cuda_check(ctx, e, call);
    int rec[4];
    e = cudaMemcpy(rec, ctx->d_err, sizeof(rec), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return clha_cuda_check(ctx, e, call);
    if (rec[0] == 0) return CLHA_OK;
    cudaMemsetAsync(ctx->d_err, 0, 4 * sizeof(int), ctx->stream);
    cudaStreamSynchronize(ctx->stream);
    return clha_fail(ctx, (clha_status)rec[0], "%s: %s reported %s (problem %d, index %d)", call,
                     kernel_name(rec[3]), status_name(rec[0]), rec[1], rec[2]);
}

#define CHECK_CTX(ctx) \
    do { if (!(ctx)) return CLHA_ERR_INVALID_ARG; } while (0)
#define REQUIRE(cond, st, ...) \
    do { if (!(cond)) return clha_fail(ctx, st, __VA_ARGS__); } while (0)
#define CUDA_TRY(expr, what) \
    do { cudaError_t e__ = (expr); if (e__ != cudaSuccess) return clha_cuda_check(ctx, e__, what); } while (0)
#define SET_DEVICE(ctx) CUDA_TRY(cudaSetDevice((ctx)->device), "cudaSetDevice")

// ------------------------------------------------------------------------------ context
extern "C" int clha_version(void) { return CLHA_VERSION; }

extern "C" clha_status clha_create(int device, void* cuda_stream, clha_ctx** out) {
    if (!out) return CLHA_ERR_INVALID_ARG;
    *out = nullptr;
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev) {
        cudaGetLastError();
        return CLHA_ERR_INVALID_ARG;
    }
    clha_ctx* ctx = new (std::nothrow) clha_ctx();
    if (!ctx) return CLHA_ERR_OOM;
    ctx->device = device;
    ctx->stream = (cudaStream_t)cuda_stream;
    if (cudaSetDevice(device) != cudaSuccess ||
        cudaDeviceGetAttribute(&ctx->num_sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess ||
        cudaMalloc(&ctx->d_err, 4 * sizeof(int)) != cudaSuccess ||
        cudaMemset(ctx->d_err, 0, 4 * sizeof(int)) != cudaSuccess ||
        cudaMalloc(&ctx->d_act_sel, sizeof(int)) != cudaSuccess ||
        cudaMemset(ctx->d_act_sel, 0, sizeof(int)) != cudaSuccess) {
        cudaGetLastError();
        if (ctx->d_err) cudaFree(ctx->d_err);
        if (ctx->d_act_sel) cudaFree(ctx->d_act_sel);
        delete ctx;
        return CLHA_ERR_CUDA;
    }
    *out = ctx;
    return CLHA_OK;
}

extern "C" void clha_destroy(clha_ctx* ctx) {
    if (!ctx) return;
    cudaSetDevice(ctx->device);
    cudaStreamSynchronize(ctx->stream);
    if (ctx->ws) cudaFree(ctx->ws);
    if (ctx->d_err) cudaFree(ctx->d_err);
    if (ctx->d_act_sel) cudaFree(ctx->d_act_sel);
    if (ctx->host_pinned) cudaFreeHost(ctx->host_pinned);
    delete ctx;
}

extern "C" const char* clha_last_error(const clha_ctx* ctx) {
    return ctx ? ctx->last_error.c_str() : "null context";
}

extern "C" clha_status clha_check(clha_ctx* ctx) {
    CHECK_CTX(ctx);
    SET_DEVICE(ctx);
    return clha_sync_and_check(ctx, "clha_check");
}

// ------------------------------------------------------------------------------ phase 1
extern "C" clha_status clha_route_topk(clha_ctx* ctx, const float* logits, int64_t n, int E, int k,
                                       int32_t* ids, int32_t* counts) {
    CHECK_CTX(ctx);
    REQUIRE(n >= 0, CLHA_ERR_INVALID_ARG, "clha_route_topk: n < 0");
    REQUIRE(E >= 1 && E <= 1024, CLHA_ERR_INVALID_ARG, "clha_route_topk: E must be in 1..1024");
    REQUIRE(k >= 1 && k <= E, CLHA_ERR_INVALID_ARG, "clha_route_topk: k must be in 1..E");
    REQUIRE(counts && (n == 0 || (logits && ids)), CLHA_ERR_INVALID_ARG, "clha_route_topk: null pointer");
    SET_DEVICE(ctx);
    LaunchScope launch_scope(ctx);
    CUDA_TRY(launch_route_topk(ctx->stream, logits, n, E, k, ids, counts, ctx->d_err), "clha_route_topk");
    return CLHA_OK;
}

extern "C" int64_t clha_packed_rows(int64_t n, int k, int E) {
    if (n < 0 || k < 1 || E < 1) return 0;
    return n * (int64_t)k + 128 * (int64_t)E;
}

static int dtype_size(clha_dtype dt) { return dt == CLHA_BF16 ? 2 : (dt == CLHA_F32 ? 4 : 0); }

extern "C" clha_status clha_gather(clha_ctx* ctx, const void* X, clha_dtype dtype, int64_t n, int d,
                                   const int32_t* ids, int k, int E, void* X_packed, int64_t packed_rows,
                                   int64_t* seg, int32_t* perm) {
    CHECK_CTX(ctx);
    int es = dtype_size(dtype);
    REQUIRE(es, CLHA_ERR_INVALID_ARG, "clha_gather: unknown dtype");
    REQUIRE(n >= 0 && d > 0, CLHA_ERR_INVALID_ARG, "clha_gather: bad sizes");
    REQUIRE(E >= 1 && E <= 1024 && k >= 1 && k <= E, CLHA_ERR_INVALID_ARG, "clha_gather: need 1 <= k <= E <= 1024");
    REQUIRE(d % 128 == 0, CLHA_ERR_UNSUPPORTED_SHAPE, "clha_gather: d=%d is not a multiple of 128", d);
    REQUIRE(packed_rows >= clha_packed_rows(n, k, E), CLHA_ERR_INVALID_ARG,
            "clha_gather: packed_rows %lld < %lld", (long long)packed_rows, (long long)clha_packed_rows(n, k, E));
    REQUIRE(seg && (X_packed || perm) && (n == 0 || ids) && (!X_packed || n == 0 || X), CLHA_ERR_INVALID_ARG,
            "clha_gather: null pointer");
    SET_DEVICE(ctx);
    LaunchScope launch_scope(ctx);
    size_t wsb = gather_workspace_bytes(n, k, E, packed_rows);
    void* ws = nullptr;
    clha_status st = clha_workspace(ctx, wsb, &ws);
    if (st) return st;
    CUDA_TRY(launch_gather(ctx->stream, X, es, n, d, ids, k, E, X_packed, packed_rows, seg, perm, ws, wsb,
                           ctx->d_err), "clha_gather");
    return CLHA_OK;
}

extern "C" clha_status clha_expert_act(clha_ctx* ctx, const void* X, int64_t rows, int d_model,
                                       const int64_t* seg, int E, const void* Wg, const void* Wu, int d_ff,
                                       void* h) {
    CHECK_CTX(ctx);
    REQUIRE(rows >= 0 && d_model > 0 && d_ff > 0 && E >= 1 && E <= 1024, CLHA_ERR_INVALID_ARG,
            "clha_expert_act: bad sizes");
    REQUIRE(seg || E == 1, CLHA_ERR_INVALID_ARG, "clha_expert_act: seg == NULL needs E == 1");
    REQUIRE(d_model % 128 == 0 && d_ff % 128 == 0, CLHA_ERR_UNSUPPORTED_SHAPE,
            "clha_expert_act: d_model=%d and d_ff=%d must be multiples of 128", d_model, d_ff);
    REQUIRE(Wg && Wu && (rows == 0 || (X && h)), CLHA_ERR_INVALID_ARG, "clha_expert_act: null pointer");
    if (rows == 0) return CLHA_OK;
    SET_DEVICE(ctx);
    LaunchScope launch_scope(ctx);
    void* ws = nullptr;
    // the tensor-core path with outlier channels needs masked weight copies: only the automatic choice
    const size_t wsb = ctx->act_policy == CLHA_ACT_AUTO ? expert_act_workspace_bytes(d_model, E, d_ff, rows) : 256;
    clha_status st = clha_workspace(ctx, wsb, &ws);
    if (st) return st;
    CUDA_TRY(launch_expert_act(ctx->stream, ctx->num_sms, (const __nv_bfloat16*)X, rows, d_model, nullptr, seg, E,
                               (const __nv_bfloat16*)Wg, (const __nv_bfloat16*)Wu, d_ff, (__nv_bfloat16*)h,
                               ctx->act_policy, ws, ctx->d_act_sel, ctx->d_err),
             "clha_expert_act");
    return CLHA_OK;
}

extern "C" clha_status clha_set_act_kernel(clha_ctx* ctx, int kernel) {
    CHECK_CTX(ctx);
    REQUIRE(kernel >= CLHA_ACT_AUTO && kernel <= CLHA_ACT_TENSOR, CLHA_ERR_INVALID_ARG,
            "clha_set_act_kernel: kernel must be CLHA_ACT_AUTO, CLHA_ACT_FMA or CLHA_ACT_TENSOR");
    ctx->act_policy = kernel;
    return CLHA_OK;
}

extern "C" int clha_last_act_kernel(clha_ctx* ctx) {
    if (!ctx) return -1;
    if (ctx->act_policy != CLHA_ACT_AUTO) return ctx->act_policy;
    int sel = 0;
    cudaSetDevice(ctx->device);
    if (cudaStreamSynchronize(ctx->stream) != cudaSuccess ||
        cudaMemcpy(&sel, ctx->d_act_sel, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) {
        cudaGetLastError();
        return -1;
    }
    return sel ? CLHA_ACT_TENSOR : CLHA_ACT_FMA;
}

extern "C" clha_status clha_expert_act_gathered(clha_ctx* ctx, const void* X, int64_t n, int d_model,
                                                const int32_t* perm, int64_t packed_rows, const int64_t* seg, int E,
                                                const void* Wg, const void* Wu, int d_ff, void* h) {
    CHECK_CTX(ctx);
    REQUIRE(n >= 0 && n < (int64_t)1 << 31 && packed_rows >= 0 && d_model > 0 && d_ff > 0 && E >= 1 && E <= 1024,
            CLHA_ERR_INVALID_ARG, "clha_expert_act_gathered: bad sizes");
    REQUIRE(d_model % 128 == 0 && d_ff % 128 == 0, CLHA_ERR_UNSUPPORTED_SHAPE,
            "clha_expert_act_gathered: d_model=%d and d_ff=%d must be multiples of 128", d_model, d_ff);
    REQUIRE(Wg && Wu && perm && seg && (packed_rows == 0 || h) && (n == 0 || X), CLHA_ERR_INVALID_ARG,
            "clha_expert_act_gathered: null pointer");
    if (packed_rows == 0 || n == 0) return CLHA_OK;
    SET_DEVICE(ctx);
    LaunchScope launch_scope(ctx);
    CUDA_TRY(launch_expert_act(ctx->stream, ctx->num_sms, (const __nv_bfloat16*)X, packed_rows, d_model, perm, seg,
                               E, (const __nv_bfloat16*)Wg, (const __nv_bfloat16*)Wu, d_ff, (__nv_bfloat16*)h,
                               CLHA_ACT_FMA, nullptr, nullptr, ctx->d_err),
             "clha_expert_act_gathered");
    return CLHA_OK;
}

extern "C" clha_status clha_accum_create(clha_ctx* ctx, int d, int n_layers, int n_slots, clha_accum** out) {
    CHECK_CTX(ctx);
    REQUIRE(out, CLHA_ERR_INVALID_ARG, "clha_accum_create: null out");
    *out = nullptr;
    REQUIRE(d > 0 && n_layers >= 1 && n_layers <= CLHA_MAX_LAYERS && n_slots >= 1, CLHA_ERR_INVALID_ARG,
            "clha_accum_create: need d > 0, 1 <= n_layers <= %d, n_slots >= 1", CLHA_MAX_LAYERS);
    REQUIRE(d % 128 == 0, CLHA_ERR_UNSUPPORTED_SHAPE, "clha_accum_create: d=%d is not a multiple of 128", d);
    SET_DEVICE(ctx);
    clha_accum* acc = new (std::nothrow) clha_accum();
    if (!acc) return CLHA_ERR_OOM;
    acc->device = ctx->device;
    acc->d = d;
    acc->n_layers = n_layers;
    acc->n_slots = n_slots;
    size_t nS = (size_t)n_layers * n_slots * d * d;
    cudaError_t e = cudaMalloc(&acc->S, nS * sizeof(float));
    if (e == cudaSuccess) e = cudaMalloc(&acc->counts, (size_t)n_layers * n_slots * sizeof(int64_t));
    if (e != cudaSuccess) {
        cudaGetLastError();
        if (acc->S) cudaFree(acc->S);
        delete acc;
        return clha_fail(ctx, CLHA_ERR_OOM, "clha_accum_create: %zu bytes", nS * sizeof(float));
    }
    *out = acc;
    return clha_accum_zero(ctx, acc);
}

extern "C" clha_status clha_accum_destroy(clha_accum* acc) {
    if (!acc) return CLHA_OK;
    cudaSetDevice(acc->device);
    cudaDeviceSynchronize();  // work still queued on any stream may reference the buffers
    cudaFree(acc->S);
    cudaFree(acc->counts);
    delete acc;
    return CLHA_OK;
}

extern "C" clha_status clha_accum_zero(clha_ctx* ctx, clha_accum* acc) {
    CHECK_CTX(ctx);
    REQUIRE(acc, CLHA_ERR_INVALID_ARG, "clha_accum_zero: null accumulator");
    SET_DEVICE(ctx);
    size_t nS = (size_t)acc->n_layers * acc->n_slots * acc->d * acc->d;
    CUDA_TRY(cudaMemsetAsync(acc->S, 0, nS * sizeof(float), ctx->stream), "clha_accum_zero");
    CUDA_TRY(cudaMemsetAsync(acc->counts, 0, (size_t)acc->n_layers * acc->n_slots * sizeof(int64_t), ctx->stream),
             "clha_accum_zero");
    return CLHA_OK;
}

extern "C" clha_status clha_accum_buffers(const clha_accum* acc, float** S, int64_t** counts) {
    if (!acc) return CLHA_ERR_INVALID_ARG;
    if (S) *S = acc->S;
    if (counts) *counts = acc->counts;
    return CLHA_OK;
}

extern "C" clha_status clha_accum_export(clha_ctx* ctx, const clha_accum* acc, float* host_S, int64_t* host_counts) {
    CHECK_CTX(ctx);
    REQUIRE(acc && host_S && host_counts, CLHA_ERR_INVALID_ARG, "clha_accum_export: null pointer");
    SET_DEVICE(ctx);
    size_t nS = (size_t)acc->n_layers * acc->n_slots * acc->d * acc->d;
    CUDA_TRY(cudaMemcpyAsync(host_S, acc->S, nS * sizeof(float), cudaMemcpyDeviceToHost, ctx->stream), "export S");
    CUDA_TRY(cudaMemcpyAsync(host_counts, acc->counts, (size_t)acc->n_layers * acc->n_slots * sizeof(int64_t),
                             cudaMemcpyDeviceToHost, ctx->stream), "export counts");
    return clha_sync_and_check(ctx, "clha_accum_export");
}

extern "C" clha_status clha_accum_import(clha_ctx* ctx, clha_accum* acc, const float* host_S, const int64_t* host_counts) {
    CHECK_CTX(ctx);
    REQUIRE(acc && host_S && host_counts, CLHA_ERR_INVALID_ARG, "clha_accum_import: null pointer");
    SET_DEVICE(ctx);
    size_t nS = (size_t)acc->n_layers * acc->n_slots * acc->d * acc->d;
    CUDA_TRY(cudaMemcpyAsync(acc->S, host_S, nS * sizeof(float), cudaMemcpyHostToDevice, ctx->stream), "import S");
    CUDA_TRY(cudaMemcpyAsync(acc->counts, host_counts, (size_t)acc->n_layers * acc->n_slots * sizeof(int64_t),
                             cudaMemcpyHostToDevice, ctx->stream), "import counts");
    return clha_sync_and_check(ctx, "clha_accum_import");
}

extern "C" clha_status clha_collect(clha_ctx* ctx, clha_accum* acc, int layer, const void* X, clha_dtype dtype,
                                    int64_t rows, int d, const int64_t* seg, int E, int slot0) {
    CHECK_CTX(ctx);
    REQUIRE(acc, CLHA_ERR_INVALID_ARG, "clha_collect: null accumulator");
    REQUIRE(dtype == CLHA_BF16 || dtype == CLHA_F32, CLHA_ERR_INVALID_ARG, "clha_collect: unknown dtype");
    REQUIRE(d == acc->d, CLHA_ERR_INVALID_ARG, "clha_collect: d=%d but the accumulator has d=%d", d, acc->d);
    REQUIRE(layer >= 0 && layer < acc->n_layers, CLHA_ERR_INVALID_ARG,
            "clha_collect: layer %d outside 0..%d (each layer has its own accumulator)", layer, acc->n_layers - 1);
    REQUIRE(rows >= 0, CLHA_ERR_INVALID_ARG, "clha_collect: rows < 0");
    int ne = seg ? E : 1;
    REQUIRE(ne >= 1 && slot0 >= 0 && slot0 + ne <= acc->n_slots, CLHA_ERR_INVALID_ARG,
            "clha_collect: slots %d..%d outside the accumulator's %d", slot0, slot0 + ne - 1, acc->n_slots);
    REQUIRE(rows == 0 || X, CLHA_ERR_INVALID_ARG, "clha_collect: null X");
    if (rows == 0) return CLHA_OK;
    SET_DEVICE(ctx);
    LaunchScope launch_scope(ctx);
    float* S_base = acc->S + ((size_t)layer * acc->n_slots + slot0) * (size_t)d * d;
    int64_t* c_base = acc->counts + (size_t)layer * acc->n_slots + slot0;
    cudaError_t e;
    if (dtype == CLHA_BF16)
        e = launch_collect_bf16(ctx->stream, ctx->num_sms, (const __nv_bfloat16*)X, rows, d, seg, ne, S_base, c_base,
                                ctx->d_err);
    else
        e = launch_collect_f32(ctx->stream, (const float*)X, rows, d, seg, ne, S_base, c_base);
    CUDA_TRY(e, "clha_collect");
    return CLHA_OK;
}

extern "C" clha_status clha_collect_gathered(clha_ctx* ctx, clha_accum* acc, int layer, const void* X, int64_t n,
                                             int d, const int32_t* perm, const int64_t* seg, int E, int slot0) {
    CHECK_CTX(ctx);
    REQUIRE(acc, CLHA_ERR_INVALID_ARG, "clha_collect_gathered: null accumulator");
    REQUIRE(d == acc->d, CLHA_ERR_INVALID_ARG, "clha_collect_gathered: d=%d but the accumulator has d=%d", d, acc->d);
    REQUIRE(layer >= 0 && layer < acc->n_layers, CLHA_ERR_INVALID_ARG,
            "clha_collect_gathered: layer %d outside 0..%d", layer, acc->n_layers - 1);
    REQUIRE(n >= 0 && n < (int64_t)1 << 31, CLHA_ERR_INVALID_ARG, "clha_collect_gathered: n outside 0 .. 2^31 - 1");
    REQUIRE(E >= 1 && slot0 >= 0 && slot0 + E <= acc->n_slots, CLHA_ERR_INVALID_ARG,
            "clha_collect_gathered: slots %d..%d outside the accumulator's %d", slot0, slot0 + E - 1, acc->n_slots);
    REQUIRE(perm && seg && (n == 0 || X), CLHA_ERR_INVALID_ARG, "clha_collect_gathered: null pointer");
    REQUIRE(((uintptr_t)perm & 15) == 0, CLHA_ERR_INVALID_ARG, "clha_collect_gathered: perm must be 16-byte aligned");
    if (n == 0) return CLHA_OK;
    SET_DEVICE(ctx);
    LaunchScope launch_scope(ctx);
    float* S_base = acc->S + ((size_t)layer * acc->n_slots + slot0) * (size_t)d * d;
    int64_t* c_base = acc->counts + (size_t)layer * acc->n_slots + slot0;
    CUDA_TRY(launch_collect_bf16_gathered(ctx->stream, ctx->num_sms, (const __nv_bfloat16*)X, n, d, perm, seg, E,
                                          S_base, c_base, ctx->d_err),
             "clha_collect_gathered");
    return CLHA_OK;
}

// ------------------------------------------------------------------------------ phase 2
extern "C" clha_status clha_aggregate(clha_ctx* ctx, const clha_accum* acc, int slot0, int n_slots,
                                      clha_alpha_mode mode, const double* alpha_in, double damp_frac,
                                      float* H_comb, float* H_damped, double* alpha_out, double* lambda_out,
                                      double* lambda_dev) {
    CHECK_CTX(ctx);
    REQUIRE(acc && H_damped, CLHA_ERR_INVALID_ARG, "clha_aggregate: null pointer");
    REQUIRE(n_slots >= 1 && slot0 >= 0 && slot0 + n_slots <= acc->n_slots, CLHA_ERR_INVALID_ARG,
            "clha_aggregate: slots outside the accumulator");
    const int amode = (int)mode & 0xff;
    REQUIRE(((int)mode & ~(0xff | CLHA_AGG_EMPTY_IDENTITY)) == 0 &&
                (amode == CLHA_ALPHA_ROUTING || amode == CLHA_ALPHA_EQUAL || amode == CLHA_ALPHA_EXPLICIT ||
                 amode == CLHA_ALPHA_SUM),
            CLHA_ERR_INVALID_ARG, "clha_aggregate: unknown alpha mode");
    REQUIRE(amode != CLHA_ALPHA_EXPLICIT || alpha_in, CLHA_ERR_INVALID_ARG, "clha_aggregate: explicit alpha needs alpha_in");
    REQUIRE(damp_frac > 0.0 && damp_frac == damp_frac, CLHA_ERR_INVALID_ARG, "clha_aggregate: damp_frac must be > 0");
    SET_DEVICE(ctx);
    LaunchScope launch_scope(ctx);
    clha_alpha_args a;
    memset(&a, 0, sizeof(a));
    a.mode = (int)mode;
    a.n_layers = acc->n_layers;
    if (amode == CLHA_ALPHA_EXPLICIT)
        for (int i = 0; i < acc->n_layers; ++i) a.alpha[i] = alpha_in[i];
    size_t need = clha_round_up((size_t)n_slots * acc->n_layers * sizeof(double)) +
                  clha_round_up((size_t)n_slots * sizeof(double));
    void* ws = nullptr;
    clha_status st = clha_workspace(ctx, need, &ws);
    if (st) return st;
    char* cur = (char*)ws;
    double* d_alpha = (double*)clha_carve(cur, (size_t)n_slots * acc->n_layers * sizeof(double));
    double* d_lambda = (double*)clha_carve(cur, (size_t)n_slots * sizeof(double));
    CUDA_TRY(launch_aggregate(ctx->stream, acc->S, acc->counts, acc->d, acc->n_layers, acc->n_slots, slot0, n_slots,
                              a, damp_frac, H_comb, H_damped, d_alpha, d_lambda, ctx->d_err),
             "clha_aggregate");
    if (lambda_dev)
        CUDA_TRY(cudaMemcpyAsync(lambda_dev, d_lambda, (size_t)n_slots * sizeof(double), cudaMemcpyDeviceToDevice,
                                 ctx->stream), "clha_aggregate lambda_dev");
    if (alpha_out || lambda_out) {
        if (alpha_out)
            CUDA_TRY(cudaMemcpyAsync(alpha_out, d_alpha, (size_t)n_slots * acc->n_layers * sizeof(double),
                                     cudaMemcpyDeviceToHost, ctx->stream), "clha_aggregate alpha");
        if (lambda_out)
            CUDA_TRY(cudaMemcpyAsync(lambda_out, d_lambda, (size_t)n_slots * sizeof(double), cudaMemcpyDeviceToHost,
                                     ctx->stream), "clha_aggregate lambda");
        return clha_sync_and_check(ctx, "clha_aggregate");
    }
    return CLHA_OK;
}

// ------------------------------------------------------------------------------ phase 3
extern "C" clha_status clha_factor_groups_as(clha_ctx* ctx, clha_factor_form form, int n_groups,
                                             const clha_factor_group* groups) {
    CHECK_CTX(ctx);
    REQUIRE(form == CLHA_FACTOR_INV_CHOL || form == CLHA_FACTOR_BLOCK_CHOL, CLHA_ERR_INVALID_ARG,
            "clha_factor: unknown form %d", (int)form);
    REQUIRE(groups, CLHA_ERR_INVALID_ARG, "clha_factor_groups: null groups");
    REQUIRE(n_groups >= 1 && n_groups <= CLHA_FACTOR_MAX_GROUPS, CLHA_ERR_INVALID_ARG,
            "clha_factor_groups: n_groups=%d outside 1..%d", n_groups, CLHA_FACTOR_MAX_GROUPS);
    FactorGroup fg[CLHA_FACTOR_MAX_GROUPS];
    for (int k = 0; k < n_groups; ++k) {
        const clha_factor_group& g = groups[k];
        REQUIRE(g.H_damped && g.U, CLHA_ERR_INVALID_ARG, "clha_factor: null pointer (group %d)", k);
        REQUIRE(g.batch >= 1 && g.d > 0, CLHA_ERR_INVALID_ARG, "clha_factor: bad sizes (group %d)", k);
        REQUIRE(g.d % 128 == 0, CLHA_ERR_UNSUPPORTED_SHAPE, "clha_factor: d=%d is not a multiple of 128 (group %d)",
                g.d, k);
        fg[k] = FactorGroup{g.H_damped, g.U, g.batch, g.d};
    }
    SET_DEVICE(ctx);
    LaunchScope launch_scope(ctx);
    void* ws = nullptr;
    clha_status st = clha_workspace(ctx, factor_workspace_bytes(fg, n_groups), &ws);
    if (st) return st;
    CUDA_TRY(launch_factor(ctx->stream, ctx->num_sms, fg, n_groups, ws, ctx->d_err, ctx->factor_wait_ns, (int)form),
             "clha_factor");
    return CLHA_OK;
}

extern "C" clha_status clha_factor_groups(clha_ctx* ctx, int n_groups, const clha_factor_group* groups) {
    return clha_factor_groups_as(ctx, CLHA_FACTOR_INV_CHOL, n_groups, groups);
}

extern "C" clha_status clha_set_factor_wait_limit(clha_ctx* ctx, uint64_t ns) {
    CHECK_CTX(ctx);
    ctx->factor_wait_ns = ns ? ns : 4000000000ull;
    return CLHA_OK;
}

extern "C" clha_status clha_factor(clha_ctx* ctx, const float* H_damped, int batch, int d, float* U) {
    clha_factor_group g{H_damped, U, batch, d};
    return clha_factor_groups(ctx, 1, &g);
}

// ------------------------------------------------------------------------------ deployable codes
extern "C" clha_status clha_pack_codes(clha_ctx* ctx, const uint8_t* codes, int64_t rows, int d_in, int bits,
                                       uint32_t* packed) {
    CHECK_CTX(ctx);
    REQUIRE(rows >= 0 && bits >= 2 && bits <= 8, CLHA_ERR_INVALID_ARG, "clha_pack_codes: need rows >= 0, 2 <= bits <= 8");
    REQUIRE(d_in > 0 && d_in % 128 == 0, CLHA_ERR_UNSUPPORTED_SHAPE, "clha_pack_codes: d_in=%d is not a multiple of 128",
            d_in);
    REQUIRE(rows == 0 || (codes && packed), CLHA_ERR_INVALID_ARG, "clha_pack_codes: null pointer");
    SET_DEVICE(ctx);
    LaunchScope launch_scope(ctx);
    CUDA_TRY(launch_pack_codes(ctx->stream, codes, rows, d_in, bits, packed), "clha_pack_codes");
    return CLHA_OK;
}

extern "C" clha_status clha_dequantize(clha_ctx* ctx, const uint32_t* packed, const float* scales,
                                       const uint8_t* zeros, int64_t rows, int d_in, int bits, float* W_hat) {
    CHECK_CTX(ctx);
    REQUIRE(rows >= 0 && bits >= 2 && bits <= 8, CLHA_ERR_INVALID_ARG, "clha_dequantize: need rows >= 0, 2 <= bits <= 8");
    REQUIRE(d_in > 0 && d_in % 128 == 0, CLHA_ERR_UNSUPPORTED_SHAPE, "clha_dequantize: d_in=%d is not a multiple of 128",
            d_in);
    REQUIRE(rows == 0 || (packed && scales && zeros && W_hat), CLHA_ERR_INVALID_ARG, "clha_dequantize: null pointer");
    SET_DEVICE(ctx);
    LaunchScope launch_scope(ctx);
    CUDA_TRY(launch_dequantize(ctx->stream, packed, scales, zeros, rows, d_in, bits, W_hat), "clha_dequantize");
    return CLHA_OK;
}

extern "C" clha_status clha_dequant_matmul(clha_ctx* ctx, const void* X, clha_dtype dtype, int64_t n,
                                           const uint32_t* packed, const float* scales, const uint8_t* zeros,
                                           int d_out, int d_in, int bits, float* Y) {
    CHECK_CTX(ctx);
    REQUIRE(dtype == CLHA_BF16 || dtype == CLHA_F32, CLHA_ERR_INVALID_ARG, "clha_dequant_matmul: unknown dtype");
    REQUIRE(n >= 0 && bits >= 2 && bits <= 8, CLHA_ERR_INVALID_ARG, "clha_dequant_matmul: need n >= 0, 2 <= bits <= 8");
    REQUIRE(d_in > 0 && d_in % 128 == 0 && d_out > 0 && d_out % 64 == 0, CLHA_ERR_UNSUPPORTED_SHAPE,
            "clha_dequant_matmul: need d_in a multiple of 128 and d_out of 64 (got %d, %d)", d_in, d_out);
    REQUIRE(n == 0 || (X && packed && scales && zeros && Y), CLHA_ERR_INVALID_ARG, "clha_dequant_matmul: null pointer");
    SET_DEVICE(ctx);
    LaunchScope launch_scope(ctx);
    CUDA_TRY(launch_dequant_matmul(ctx->stream, X, dtype == CLHA_BF16, n, d_in, packed, scales, zeros, d_out, bits, Y),
             "clha_dequant_matmul");
    return CLHA_OK;
}

extern "C" clha_status clha_routing_divergence(clha_ctx* ctx, const int64_t* counts, int n_layers, int ld,
                                               int slot0, int E, double* tv) {
    CHECK_CTX(ctx);
    REQUIRE(counts && tv, CLHA_ERR_INVALID_ARG, "clha_routing_divergence: null pointer");
    REQUIRE(n_layers >= 1 && n_layers <= CLHA_DIVERGENCE_MAX_LAYERS && E >= 1 && slot0 >= 0 && ld >= 1 &&
                (int64_t)slot0 + E <= ld,
            CLHA_ERR_INVALID_ARG, "clha_routing_divergence: need 1 <= n_layers <= %d, E >= 1, 0 <= slot0, slot0 + E <= ld",
            CLHA_DIVERGENCE_MAX_LAYERS);
    SET_DEVICE(ctx);
    LaunchScope launch_scope(ctx);
    CUDA_TRY(launch_routing_divergence(ctx->stream, counts, n_layers, ld, slot0, E, tv, ctx->d_err),
             "clha_routing_divergence");
    return CLHA_OK;
}

extern "C" clha_status clha_epmq_target(clha_ctx* ctx, const clha_accum* acc, int slot, const void* W_src,
                                        const void* W_merged, clha_dtype dtype, int d_out, const float* U,
                                        const double* lambda_dev, float* W_target) {
    CHECK_CTX(ctx);
    REQUIRE(acc && W_src && W_merged && U && lambda_dev && W_target, CLHA_ERR_INVALID_ARG,
            "clha_epmq_target: null pointer");
    REQUIRE(dtype == CLHA_BF16 || dtype == CLHA_F32, CLHA_ERR_INVALID_ARG, "clha_epmq_target: unknown dtype");
    REQUIRE(slot >= 0 && slot < acc->n_slots, CLHA_ERR_INVALID_ARG, "clha_epmq_target: slot %d outside 0..%d", slot,
            acc->n_slots - 1);
    REQUIRE(d_out > 0 && d_out % 64 == 0, CLHA_ERR_UNSUPPORTED_SHAPE,
            "clha_epmq_target: d_out=%d is not a positive multiple of 64", d_out);
    SET_DEVICE(ctx);
    LaunchScope launch_scope(ctx);
    void* ws = nullptr;
    const int d = acc->d;
    clha_status st = clha_workspace(ctx, epmq_workspace_bytes(d_out, d), &ws);
    if (st) return st;
    const int64_t dd = (int64_t)d * d;
    CUDA_TRY(launch_epmq_target(ctx->stream, acc->S + (size_t)slot * dd, (int64_t)acc->n_slots * dd, acc->n_layers,
                                W_src, dtype == CLHA_BF16, W_merged, d_out, d, U, lambda_dev, W_target, ws),
             "clha_epmq_target");
    return CLHA_OK;
}

extern "C" clha_status clha_quantize_as(clha_ctx* ctx, clha_factor_form form, const float* U, int n_u, const void* W,
                                        clha_dtype dtype, int batch, int d_out, int d_in, const clha_quant_params* p,
                                        uint8_t* codes, float* scales, uint8_t* zeros, float* W_hat,
                                        const double* lambda, double* loss) {
    CHECK_CTX(ctx);
    REQUIRE(form == CLHA_FACTOR_INV_CHOL || form == CLHA_FACTOR_BLOCK_CHOL, CLHA_ERR_INVALID_ARG,
            "clha_quantize: unknown factor form %d", (int)form);
    REQUIRE(U && W && p && codes && scales && zeros, CLHA_ERR_INVALID_ARG, "clha_quantize: null pointer");
    REQUIRE(dtype == CLHA_BF16 || dtype == CLHA_F32, CLHA_ERR_INVALID_ARG, "clha_quantize: unknown dtype");
    REQUIRE(batch >= 1 && d_out > 0 && d_in > 0 && n_u >= 1 && n_u <= batch, CLHA_ERR_INVALID_ARG,
            "clha_quantize: bad sizes (need batch >= 1, 1 <= n_u <= batch)");
    REQUIRE(p->bits >= 2 && p->bits <= 8, CLHA_ERR_INVALID_ARG, "clha_quantize: bits=%d outside 2..8", p->bits);
    REQUIRE(d_in % 128 == 0 && d_out % 128 == 0, CLHA_ERR_UNSUPPORTED_SHAPE,
            "clha_quantize: d_out=%d and d_in=%d must be multiples of 128", d_out, d_in);
    REQUIRE((lambda == nullptr) == (loss == nullptr), CLHA_ERR_INVALID_ARG,
            "clha_quantize: lambda and loss go together (both or neither)");
    REQUIRE(p->group == 128 && p->block == 128, CLHA_ERR_UNSUPPORTED_SHAPE,
            "clha_quantize: group=%d block=%d (supported: 128, 128)", p->group, p->block);
    SET_DEVICE(ctx);
    LaunchScope launch_scope(ctx);
    void* ws = nullptr;
    clha_status st = clha_workspace(ctx, quantize_workspace_bytes(batch, d_out, d_in), &ws);
    if (st) return st;
    CUDA_TRY(launch_quantize(ctx->stream, ctx->num_sms, U, n_u, W, dtype == CLHA_F32, batch, d_out, d_in, p->bits, codes,
                             scales, zeros, W_hat, lambda, loss, ws, ctx->d_err, (int)form), "clha_quantize");
    return CLHA_OK;
}

extern "C" clha_status clha_quantize(clha_ctx* ctx, const float* U, int n_u, const void* W, clha_dtype dtype,
                                     int batch, int d_out, int d_in, const clha_quant_params* p,
                                     uint8_t* codes, float* scales, uint8_t* zeros, float* W_hat,
                                     const double* lambda, double* loss) {
    return clha_quantize_as(ctx, CLHA_FACTOR_INV_CHOL, U, n_u, W, dtype, batch, d_out, d_in, p, codes, scales, zeros,
                            W_hat, lambda, loss);
}

extern "C" clha_status clha_loss(clha_ctx* ctx, const void* W, clha_dtype dtype, const float* W_hat, const float* H,
                                 int n_h, int batch, int d_out, int d_in, double* loss_out) {
    CHECK_CTX(ctx);
    REQUIRE(W && W_hat && H && loss_out, CLHA_ERR_INVALID_ARG, "clha_loss: null pointer");
    REQUIRE(dtype == CLHA_BF16 || dtype == CLHA_F32, CLHA_ERR_INVALID_ARG, "clha_loss: unknown dtype");
    REQUIRE(batch >= 1 && d_out > 0 && d_in > 0 && n_h >= 1 && n_h <= batch, CLHA_ERR_INVALID_ARG,
            "clha_loss: bad sizes (need batch >= 1, 1 <= n_h <= batch)");
    REQUIRE(d_in % 128 == 0 && d_out % 128 == 0, CLHA_ERR_UNSUPPORTED_SHAPE,
            "clha_loss: d_out=%d and d_in=%d must be multiples of 128", d_out, d_in);
    SET_DEVICE(ctx);
    LaunchScope launch_scope(ctx);
    void* ws = nullptr;
    clha_status st = clha_workspace(ctx, (size_t)batch * sizeof(double), &ws);
    if (st) return st;
    double* d_loss = (double*)ws;
    CUDA_TRY(cudaMemsetAsync(d_loss, 0, (size_t)batch * sizeof(double), ctx->stream), "clha_loss");
    CUDA_TRY(launch_loss(ctx->stream, W, dtype == CLHA_F32, W_hat, H, n_h, batch, d_out, d_in, d_loss), "clha_loss");
    CUDA_TRY(cudaMemcpyAsync(loss_out, d_loss, (size_t)batch * sizeof(double), cudaMemcpyDeviceToHost, ctx->stream),
             "clha_loss copy");
    return clha_sync_and_check(ctx, "clha_loss");
}


// ------------------------------------------------------------------------------ multi-GPU exchange
extern "C" clha_status clha_pack_upper(clha_ctx* ctx, const float* S, int64_t n_outer, int64_t outer_stride,
                                       int64_t n_inner, int d, float* packed) {
    CHECK_CTX(ctx);
    REQUIRE(n_outer >= 0 && n_inner >= 0 && d > 0 && outer_stride >= n_inner, CLHA_ERR_INVALID_ARG,
            "clha_pack_upper: bad sizes (need n_outer, n_inner >= 0, d > 0, outer_stride >= n_inner)");
    REQUIRE((S && packed) || n_outer * n_inner == 0, CLHA_ERR_INVALID_ARG, "clha_pack_upper: null pointer");
    SET_DEVICE(ctx);
    LaunchScope launch_scope(ctx);
    CUDA_TRY(launch_pack_upper(ctx->stream, S, n_outer, outer_stride, n_inner, d, packed), "clha_pack_upper");
    return CLHA_OK;
}

extern "C" clha_status clha_unpack_upper(clha_ctx* ctx, const float* packed, int64_t n_outer, int64_t outer_stride,
                                         int64_t n_inner, int d, float* S) {
    CHECK_CTX(ctx);
    REQUIRE(n_outer >= 0 && n_inner >= 0 && d > 0 && outer_stride >= n_inner, CLHA_ERR_INVALID_ARG,
            "clha_unpack_upper: bad sizes (need n_outer, n_inner >= 0, d > 0, outer_stride >= n_inner)");
    REQUIRE((S && packed) || n_outer * n_inner == 0, CLHA_ERR_INVALID_ARG, "clha_unpack_upper: null pointer");
    SET_DEVICE(ctx);
    LaunchScope launch_scope(ctx);
    CUDA_TRY(launch_unpack_upper(ctx->stream, packed, n_outer, outer_stride, n_inner, d, S), "clha_unpack_upper");
    return CLHA_OK;
}
