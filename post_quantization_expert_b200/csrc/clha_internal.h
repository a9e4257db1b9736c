// Internal declarations shared by the CUDA translation units of libclha.so.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <string>

#include "clha.h"

struct clha_ctx {
    int device = 0;
    cudaStream_t stream = nullptr;
    int num_sms = 148;
    std::string last_error;
    // Device error record written by kernels: [0] status code (0 = none), [1] problem index,
    // [2] column / element index, [3] kernel id. Read and cleared by synchronising calls.
    int* d_err = nullptr;
    // Grow-only workspace.
    void* ws = nullptr;
    size_t ws_bytes = 0;
    // Kernels launched through this context (tracing).
    int64_t launches = 0;
    // Expert activation: kernel policy (0 chosen per call on the device, 1 fp32 FMA, 2 tensor cores)
    // and the device int the per-call choice is written to.
    int act_policy = 0;
    int* d_act_sel = nullptr;
    // Time limit of each dependency wait inside the factor graph (clha_set_factor_wait_limit).
    uint64_t factor_wait_ns = 4000000000ull;
    // Small pinned host buffer for scalar read-backs.
    void* host_pinned = nullptr;
    size_t host_pinned_bytes = 0;
};

struct clha_accum {
    int device = 0;
    int d = 0, n_layers = 0, n_slots = 0;
    float* S = nullptr;        // [n_layers][n_slots][d][d]
    int64_t* counts = nullptr; // [n_layers][n_slots]
};

enum clha_kernel_id {
    KID_ROUTE = 1, KID_GATHER = 2, KID_ACT = 3, KID_COLLECT = 4, KID_AGGREGATE = 5,
    KID_FACTOR = 6, KID_QUANTIZE = 7, KID_LOSS = 8, KID_DIVERGENCE = 9
};

// ------------------------------------------------------------------------------ device helpers
__device__ __forceinline__ void clha_record_error(int* err, int code, int problem, int index, int kid) {
    if (atomicCAS(err, 0, code) == 0) {
        err[1] = problem;
        err[2] = index;
        err[3] = kid;
        __threadfence();
    }
}

// ------------------------------------------------------------------------------ host helpers
clha_status clha_fail(clha_ctx* ctx, clha_status st, const char* fmt, ...);
clha_status clha_cuda_check(clha_ctx* ctx, cudaError_t e, const char* what);
// Workspace of at least `bytes` (grows; synchronises the stream when it has to reallocate).
clha_status clha_workspace(clha_ctx* ctx, size_t bytes, void** out);
// Carve an aligned sub-buffer out of a workspace cursor.
inline void* clha_carve(char*& cur, size_t bytes) {
    void* p = cur;
    cur += (bytes + 255) & ~size_t(255);
    return p;
}
inline size_t clha_round_up(size_t b) { return (b + 255) & ~size_t(255); }
// Synchronise and turn a recorded device error into a status (and clear it).
clha_status clha_sync_and_check(clha_ctx* ctx, const char* call);
// Check the last launch of a kernel.
clha_status clha_launch_check(clha_ctx* ctx, const char* what);

// Process-wide count of kernel launches (each launcher notes its launches; the API adds the
// difference to the calling context's counter).
void clha_note_launches(int n);
int64_t clha_total_launches();

// ------------------------------------------------------------------------------ kernel launchers
// Each returns cudaSuccess or the launch error; argument validation happens in api.cu.
cudaError_t launch_route_topk(cudaStream_t s, const float* logits, int64_t n, int E, int k,
                              int32_t* ids, int32_t* counts, int* err);
cudaError_t launch_gather(cudaStream_t s, const void* X, int esize, int64_t n, int d,
                          const int32_t* ids, int k, int E, void* X_packed, int64_t packed_rows,
                          int64_t* seg, int32_t* perm, void* ws, size_t ws_bytes, int* err);
size_t gather_workspace_bytes(int64_t n, int k, int E, int64_t packed_rows);
constexpr int kGatherBlockTokens = 256;   // tokens per block of the histogram and scatter passes
// Outlier channels (max |x| above 4x the channels' mean) the tensor-core activation takes out of its
// tensor-core sums and adds exactly in its epilogue; more than this and the fp32-FMA kernel runs.
constexpr int kMaxOutliers = 64;
size_t expert_act_workspace_bytes(int d_model, int E, int d_ff, int64_t rows);
cudaError_t launch_expert_act(cudaStream_t s, int num_sms, const __nv_bfloat16* X, int64_t rows, int d_model,
                              const int32_t* perm, const int64_t* seg, int E, const __nv_bfloat16* Wg,
                              const __nv_bfloat16* Wu, int d_ff, __nv_bfloat16* h, int policy, void* ws, int* sel,
                              int* err);
cudaError_t launch_expert_act_tc(cudaStream_t s, int num_sms, const __nv_bfloat16* X, int64_t rows, int d_model,
                                 const int64_t* seg, int E, const __nv_bfloat16* Wg, const __nv_bfloat16* Wu, int d_ff,
                                 __nv_bfloat16* h, const int* sel, const __nv_bfloat16* Wgm, const __nv_bfloat16* Wum,
                                 const int* out_n, const float* xo, const float* wo, int* err);
cudaError_t launch_collect_bf16_gathered(cudaStream_t s, int num_sms, const __nv_bfloat16* X, int64_t n, int d,
                                         const int32_t* perm, const int64_t* seg, int E, float* S_base,
                                         int64_t* counts_base, int* err);
cudaError_t launch_collect_bf16(cudaStream_t s, int num_sms, const __nv_bfloat16* X, int64_t rows, int d,
                                const int64_t* seg, int E, float* S_base, int64_t* counts_base,
                                int* err);
cudaError_t launch_collect_f32(cudaStream_t s, const float* X, int64_t rows, int d,
                               const int64_t* seg, int E, float* S_base, int64_t* counts_base);
struct clha_alpha_args {
    int mode;             // clha_alpha_mode
    int n_layers;
    double alpha[CLHA_MAX_LAYERS];   // explicit weights
};
cudaError_t launch_aggregate(cudaStream_t s, const float* S, const int64_t* counts, int d,
                             int n_layers, int n_slots_total, int slot0, int n_slots,
                             clha_alpha_args a, double damp_frac, float* H_comb, float* H_d,
                             double* d_alpha, double* d_lambda, int* err);
struct FactorGroup {
    const float* H;
    float* U;
    int batch, d;
};
size_t factor_workspace_bytes(const FactorGroup* groups, int n);
// form 0: U (H_d^-1 = U^T U); form 1: F, the block-scaled Cholesky factor of H_d (factor.cu)
cudaError_t launch_factor(cudaStream_t s, int num_sms, const FactorGroup* groups, int n, void* ws, int* err,
                          uint64_t wait_ns, int form);
cudaError_t launch_pack_codes(cudaStream_t s, const uint8_t* codes, int64_t rows, int d_in, int bits,
                              uint32_t* packed);
cudaError_t launch_dequantize(cudaStream_t s, const uint32_t* packed, const float* scales, const uint8_t* zeros,
                              int64_t rows, int d_in, int bits, float* W_hat);
cudaError_t launch_dequant_matmul(cudaStream_t s, const void* X, int x_bf16, int64_t n, int d_in,
                                  const uint32_t* packed, const float* scales, const uint8_t* zeros, int d_out, int bits,
                                  float* Y);
cudaError_t launch_routing_divergence(cudaStream_t s, const int64_t* counts, int L, int ld, int slot0, int E,
                                      double* tv, int* err);
size_t epmq_workspace_bytes(int d_out, int d);
cudaError_t launch_epmq_target(cudaStream_t s, const float* S_slot, int64_t layer_stride, int K, const void* W_src,
                               int w_bf16, const void* W_m, int d_out, int d, const float* U, const double* lambda,
                               float* W_target, void* ws);
cudaError_t launch_pack_upper(cudaStream_t s, const float* S, int64_t n_outer, int64_t outer_stride, int64_t n_inner,
                              int d, float* P);
cudaError_t launch_unpack_upper(cudaStream_t s, const float* P, int64_t n_outer, int64_t outer_stride,
                                int64_t n_inner, int d, float* S);
size_t quantize_workspace_bytes(int batch, int d_out, int d_in);
cudaError_t launch_quantize(cudaStream_t s, int num_sms, const float* U, int n_u, const void* W, int w_is_f32,
                            int batch, int d_out, int d_in, int bits, uint8_t* codes, float* scales,
                            uint8_t* zeros, float* W_hat, const double* lambda, double* loss, void* ws,
                            int* err, int form);   // form as launch_factor's: the factor U holds
cudaError_t launch_loss(cudaStream_t s, const void* W, int w_is_f32, const float* W_hat, const float* H,
                        int n_h, int batch, int d_out, int d_in, double* d_loss);
