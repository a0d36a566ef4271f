// Internal declarations shared by the translation units of libmla.so.
// Nothing here is part of the C ABI (that is include/mla.h).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "mla.h"
#include "mla_rope.cuh"

namespace mla {

// Problem description after host-side validation.
struct Problem {
    int H, d_c, d_r, d_n, d_v;
    int dtype;  // MLA_DTYPE_*
    float rope_base;
    float scale;  // softmax scale (already resolved)
    int B, q_len;
    RopeTable rope;  // inverse RoPE frequencies (fp64, host-computed)
};

// Optional stage-boundary events of one decode call (see MLA_EV_* in mla.h).
struct Events {
    cudaEvent_t ev[MLA_NUM_EVENTS];
    bool on = false;
    void record(int i, cudaStream_t st) const {
        if (on) cudaEventRecord(ev[i], st);
    }
};

struct CacheView {
    void* data;
    int T_max;
    int64_t stride_b, stride_t;  // elements
};

// 16-byte-aligned carving of the caller's workspace.
struct Carve {
    char* base;
    size_t off;
    explicit Carve(void* p) : base(static_cast<char*>(p)), off(0) {}
    void* take(size_t bytes) {
        void* r = base ? base + off : nullptr;
        off += (bytes + 255) & ~size_t(255);
        return r;
    }
};

// Records the thread's last-error text (read by mla_last_error) and returns `code`.
int set_error(int code, const char* fmt, ...);

// Device status word of the current device (set up once per device).
int* device_status_ptr();

// Number of SMs of the current device.
int device_sm_count();

// ----------------------------------------------------------- generic CUDA path
// Plain CUDA-core kernels, any head geometry, fp32 or bf16 storage.
cudaError_t generic_append(const Problem& p, const void* c_kv, const void* k_rope, const int32_t* pos,
                           int n_tok, const CacheView& cache, int* status, cudaStream_t st);
cudaError_t generic_absorb(const Problem& p, const void* q_nope, const void* q_rope, const void* W_UK,
                           const int32_t* seqlens, void* q_hat, cudaStream_t st);
cudaError_t generic_attend(const Problem& p, const void* q_hat, const CacheView& cache,
                           const int32_t* seqlens, void* o_lat, int* status, cudaStream_t st);
cudaError_t generic_project(const Problem& p, const void* o_lat, const void* W_UV, int rows, void* out,
                            cudaStream_t st);
size_t generic_workspace_bytes(const Problem& p);

// ----------------------------------------------------------- sm_100a path
// bf16 storage, V3 head geometry (d_c 512, d_r 64, d_n 128, d_v 128), H = 128.
bool sm100_supported(const Problem& p, int q_len);
cudaError_t sm100_append(const Problem& p, const void* c_kv, const void* k_rope, const int32_t* pos,
                         int n_tok, const CacheView& cache, int* status, cudaStream_t st);
// When given, the absorb GEMM also writes the attention's split plan.
struct PlanRequest {
    void* plan;   // start of the attention workspace
    void* o_lat;  // zeroed for sequences with an invalid length
    int T_max, clusters, overhead_tiles, min_tiles;
};
cudaError_t sm100_absorb(const Problem& p, const void* q_nope, const void* q_rope, const void* W_UK,
                         const int32_t* seqlens, void* q_hat, cudaStream_t st, const PlanRequest* plan = nullptr);
cudaError_t sm100_attend(const Problem& p, const void* q_hat, const CacheView& cache, const int32_t* seqlens,
                         void* o_lat, void* workspace, size_t ws_bytes, int num_pairs, int overhead_tiles,
                         int min_tiles, int* status, cudaStream_t st, const Events* events = nullptr,
                         bool plan_ready = false, bool combine = true, const void* prefetch = nullptr,
                         size_t prefetch_bytes = 0, const mla_decode_opts_t* opts = nullptr);
cudaError_t sm100_project(const Problem& p, const void* o_lat, const void* W_UV, int rows, void* out,
                          cudaStream_t st);
// Small batches: matrix-vector kernels.  The project step (B * q_len <= 8)
// reads the attention workspace and merges split partials itself (the
// attention step then runs without its combine kernel); the absorb step
// uses them up to 2 rows, the tensor-core GEMM above.
constexpr int kSmallRows = 8;
constexpr int kSmallAbsorbRows = 2;
cudaError_t sm100_absorb_small(const Problem& p, const void* q_nope, const void* q_rope, const void* W_UK,
                               const int32_t* seqlens, void* q_hat, cudaStream_t st, const PlanRequest* plan);
cudaError_t sm100_project_small(const Problem& p, void* attend_workspace, int num_pairs, const void* o_lat,
                                const void* W_UV, void* out, cudaStream_t st);
size_t sm100_attend_workspace_bytes(const Problem& p, int num_pairs);
// Projections around the attention step (bf16, V3 geometry): the cache append
// from the block input and the output projection.
bool sm100_linear_supported(const Problem& p);
size_t append_hidden_workspace(int rows, int d_model);
size_t output_projection_workspace(const Problem& p, int rows, int d_model);
cudaError_t sm100_append_hidden(const Problem& p, const void* x, const void* W_A, const void* gamma,
                                const int32_t* pos, int n_tok, int d_model, const CacheView& cache, void* ws,
                                int* status, cudaStream_t st);
cudaError_t sm100_output_projection(const Problem& p, const void* attn_out, const void* W_O, int rows, int d_model,
                                    void* y, void* ws, int* status, cudaStream_t st);
int sm100_default_pairs();

}  // namespace mla
