/*
 * mla.h -- C ABI of libmla.so: absorbed Multi-head Latent Attention (MLA)
 * decode on NVIDIA B200 (sm_100a).
 *
 * The method (DeepSeek-V3 MLA, decode step, absorbed order):
 *   - per token and layer the cache keeps only a latent c_KV (d_c = 512) and a
 *     decoupled RoPE key k_R (d_r = 64), 576 numbers
 *     (wq-win.github.io/llm/092-deepseekv3.html, section 二 "MLA：缓存压缩后的历史";
 *      ailearn.mscapital.top/deepseek-v3.html, MLA paragraph after the
 *      configuration table);
 *   - each head's content query is folded through W_UK into latent space and
 *     dotted with every cached c_KV; the RoPE score q_R . k_R is added
 *     separately (092 page, section 二 "缓存压缩也可以做一个代数检查":
 *      q^T (U c) = (U^T q)^T c; m.lsln.cn/news/222502 sections 2.2 and 2.3);
 *   - softmax over the whole history, aggregate sum_j p_j c_KV,j in latent
 *     space, then map through W_UV to the per-head output
 *     (ailearn.mscapital.top/deepseek-v3.html, MLA "状态传导图" panel).
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers unless stated otherwise; the
 *     caller owns every buffer, and the library keeps no pointer after a call
 *     returns.  Tensors are dense and row-major in the layouts given below.
 *   - dtype: MLA_DTYPE_BF16 (storage bf16, fp32 accumulation) or
 *     MLA_DTYPE_F32.  Every tensor of one call has the call's dtype, except
 *     positions / seqlens (int32) and the workspace (bytes).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) and never synchronise the host, except
 *     mla_device_status().
 *   - Return value: MLA_OK (0) or a negative MLA_ERR_* code.  On error nothing
 *     was launched and mla_last_error() (thread-local) describes why.
 *   - Values that live on the device (positions, seqlens) are checked by the
 *     kernels: a bad value sets a bit in the library's device status word and
 *     the affected rows are skipped (append) or written as zeros (decode);
 *     mla_device_status() reports and clears the word.
 *   - Pointers must be 16-byte aligned (MLA_ERR_ALIGN otherwise).
 */
#ifndef MLA_H_
#define MLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* mla_stream_t; /* same type as cudaStream_t */

enum {
    MLA_OK = 0,
    MLA_ERR_ARG = -1,         /* NULL pointer, negative size, bad enum */
    MLA_ERR_SHAPE = -2,       /* dimensions outside what an entry point supports */
    MLA_ERR_ALIGN = -3,       /* pointer or stride not 16-byte aligned */
    MLA_ERR_CUDA = -4,        /* a CUDA runtime/driver call failed */
    MLA_ERR_TIMEOUT = -5,     /* a device-side wait gave up (see mla_device_status) */
    MLA_ERR_DEVICE = -6,      /* device status word non-zero (bad positions/seqlens) */
    MLA_ERR_WORKSPACE = -7,   /* workspace NULL or smaller than mla_workspace_bytes() */
    MLA_ERR_UNSUPPORTED = -8  /* a forced path cannot run this shape / device */
};

enum { MLA_DTYPE_BF16 = 0, MLA_DTYPE_F32 = 1 };

/* Head geometry.  V3 values: H=128, d_c=512, d_r=64, d_n=128, d_v=128
 * (ailearn.mscapital.top/deepseek-v3.html, configuration table, row "MLA").
 * rope_base: RoPE frequency base (10000).  softmax_scale: 0 selects
 * 1/sqrt(d_n + d_r). */
typedef struct {
    int32_t H, d_c, d_r, d_n, d_v;
    int32_t dtype;
    float rope_base;
    float softmax_scale;
} mla_dims_t;

/* The compressed KV cache: B sequences x T_max rows; row t of sequence b
 * starts at data + b*stride_b + t*stride_t (strides in ELEMENTS) and holds
 * d_c latent values followed by d_r RoPE-key values already rotated at
 * position t.  stride_t >= d_c + d_r; strides*elem_size multiples of 16. */
typedef struct {
    void* data;
    int32_t B, T_max;
    int64_t stride_b, stride_t;
} mla_cache_t;

/* Device status bits (mla_device_status). */
enum {
    MLA_STATUS_BAD_POS = 1,     /* append: pos[b] < 0 or pos[b] + n_tok > T_max */
    MLA_STATUS_BAD_SEQLEN = 2,  /* decode: seqlens[b] < q_len or > T_max */
    MLA_STATUS_TIMEOUT = 4      /* a bounded device-side wait expired */
};

/* ---------------------------------------------------------------- a1: append
 * Write n_tok new tokens per sequence into the cache (092 page, section 二
 * "MLA：缓存压缩后的历史": the cache keeps c_KV and the RoPE key).
 *   c_kv   [B][n_tok][d_c]   latent of each new token
 *   k_rope [B][n_tok][d_r]   UN-rotated RoPE key; rotated here at its position
 *   pos    [B] int32         position of the first new token of sequence b
 * Row pos[b]+i of sequence b becomes [c_kv[b][i] || RoPE(k_rope[b][i], pos[b]+i)].
 * Rows with an out-of-range position are skipped and flag MLA_STATUS_BAD_POS. */
int mla_append_cache(const mla_dims_t* dims, const void* c_kv, const void* k_rope,
                     const int32_t* pos, int32_t B, int32_t n_tok,
                     const mla_cache_t* cache, mla_stream_t stream);

/* Bytes of scratch mla_decode / mla_attend_latent need for this shape on the
 * current device (depends on the SM count, not on the sequence lengths). */
size_t mla_workspace_bytes(const mla_dims_t* dims, int32_t B, int32_t q_len);

/* ---------------------------------------------------------------- decode
 * One absorbed-MLA decode step for B sequences with q_len query tokens each
 * (q_len = 1 plain decode; 2..16 speculative verify, causal among the new
 * tokens).  seqlens[b] counts cached tokens INCLUDING the q_len new ones,
 * which must already be appended; query i sits at position
 * m = seqlens[b] - q_len + i and attends to keys 0..m.
 *   q_nope [B][q_len][H][d_n]   content query
 *   q_rope [B][q_len][H][d_r]   UN-rotated RoPE query (rotated here at m)
 *   W_UK   [H][d_n][d_c]        k_C = W_UK[h] c      (U in R^{d_h x d_c})
 *   W_UV   [H][d_v][d_c]        v   = W_UV[h] c
 *   out    [B][q_len][H][d_v]   written
 *   workspace: device scratch of at least mla_workspace_bytes(), 16-byte
 *   aligned; the library rounds its base up to 256 bytes inside the buffer
 *   (mla_workspace_bytes() includes that slack).  The call owns it until the
 *   stream reaches the end of the call.
 * Steps: absorb (a2), attend in latent space (a3+a4), project (a5). */
int mla_decode(const mla_dims_t* dims, const void* q_nope, const void* q_rope,
               const void* W_UK, const void* W_UV, const mla_cache_t* cache,
               const int32_t* seqlens, int32_t B, int32_t q_len, void* out,
               void* workspace, size_t workspace_bytes, mla_stream_t stream);

/* Execution options for tests, tuning and profiling.
 *   path: 0 = auto (sm_100a tensor-core kernels for bf16 V3 geometry, generic
 *         CUDA kernels otherwise), 1 = force the tensor-core path
 *         (MLA_ERR_UNSUPPORTED if it cannot run), 2 = force the generic path.
 *   num_pairs: CTA pairs (clusters) of the attention grid (0 = one per two SMs;
 *         larger values are capped to that, the clusters that fit on the
 *         device at once, for which mla_workspace_bytes() sizes the scratch).
 *   overhead_tiles: scheduling cost charged per query token (each of the
 *         B * q_len tokens is scheduled on its own), in 64-key tiles
 *         (negative = default, 2).
 *   min_tiles: smallest piece of a token's keys one cluster takes, in 64-key tiles
 *         (0 = default, 2); larger values mean fewer split partials to merge.
 *         A batch whose sequences all have the same length is cut at sequence
 *         boundaries when that costs at most a quarter more per cluster group
 *         than an even split.
 *   events / n_events: optional caller-created cudaEvent_t handles; when
 *         n_events >= MLA_NUM_EVENTS, mla_decode_ex records them on `stream`
 *         at the stage boundaries listed below, so a caller can time each
 *         kernel with cudaEventElapsedTime.  The library does not own them.
 *   wait_limit_ns: time limit of each device-side barrier wait of the
 *         attention kernel (0 = default, 2 s).  A wait that runs out sets
 *         MLA_STATUS_TIMEOUT; the kernel then stops, drains what it has in
 *         flight and exits, leaving the context usable.
 *   withhold_tile: test hook for that path; 0 = off.  A value k > 0 makes
 *         the attention kernel's loader stop before the k-th 64-key tile of
 *         each cluster, so a bounded wait runs out and the call reports
 *         MLA_STATUS_TIMEOUT (the result is then undefined).
 *   All-zero options are valid (overhead_tiles 0 charges nothing per sequence). */
typedef struct {
    int32_t path;
    int32_t num_pairs;
    int32_t overhead_tiles;
    int32_t min_tiles;
    int32_t n_events;
    void* const* events;
    int64_t wait_limit_ns;
    int32_t withhold_tile;
    int32_t reserved;
} mla_decode_opts_t;

/* Event slots recorded by mla_decode_ex (sm_100a path; the generic path
 * records 0, 1 before/after absorb and 5 at the end, with 2..4 after attend). */
enum {
    MLA_EV_START = 0,        /* before the absorb GEMM */
    MLA_EV_ABSORB_DONE = 1,  /* after absorb (before the split planner) */
    MLA_EV_ATTEND_BEGIN = 2, /* before the attention kernel */
    MLA_EV_ATTEND_END = 3,   /* after the attention kernel (before the split combine) */
    MLA_EV_COMBINE_DONE = 4, /* after the split combine (before W_UV) */
    MLA_EV_END = 5,          /* after the W_UV projection */
    MLA_NUM_EVENTS = 6
};

int mla_decode_ex(const mla_dims_t* dims, const void* q_nope, const void* q_rope,
                  const void* W_UK, const void* W_UV, const mla_cache_t* cache,
                  const int32_t* seqlens, int32_t B, int32_t q_len, void* out,
                  void* workspace, size_t workspace_bytes,
                  const mla_decode_opts_t* opts, mla_stream_t stream);

/* ---------------------------------------------------------------- no-allocation decode
 * The same decode step as mla_decode for callers that cannot allocate device
 * memory: code whose device memory is owned by another allocator (a server or
 * framework that does not let plug-ins call cudaMalloc), or a serving loop
 * that must not allocate after start-up because cudaMalloc / cudaFree can
 * synchronise the device.  The paper has no counterpart; this is an
 * interface convenience of this library.
 *
 * Arguments, layouts and results are those of mla_decode, without the
 * workspace: the scratch is a fixed 64 MiB array inside the library's device
 * image, which every GPU that loads the library keeps until the process
 * exits.  A batch whose mla_workspace_bytes() exceeds 64 MiB is rejected with
 * MLA_ERR_WORKSPACE before anything is launched; on a 148-SM B200 the limit
 * is B * q_len <= 88 query tokens (88 sequences at q_len = 1, 44 at
 * q_len = 2, 22 at q_len = 4).  The call allocates nothing
 * and calls no allocating routine.
 *
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current); make that first call
 * before any stream capture.  All calls on a device share the one array and
 * it keeps the last call's contents (nothing needs to start at zero); calls
 * that overlap on the GPU, on different streams or threads, race on it and
 * must be ordered by the caller. */
int mla_decode_no_alloc(const mla_dims_t* dims, const void* q_nope, const void* q_rope,
                        const void* W_UK, const void* W_UV, const mla_cache_t* cache,
                        const int32_t* seqlens, int32_t B, int32_t q_len, void* out,
                        mla_stream_t stream);

/* ---------------------------------------------------------------- steps
 * The three stages of mla_decode, callable one by one (same layouts).
 *
 * a2: q_hat[b][i][h] = [ W_UK[h]^T q_nope[b][i][h]  ||  RoPE(q_rope[b][i][h], m) ]
 *     q_hat [B][q_len][H][d_c + d_r], dtype of the call. */
int mla_absorb_query(const mla_dims_t* dims, const void* q_nope, const void* q_rope,
                     const void* W_UK, const int32_t* seqlens, int32_t B, int32_t q_len,
                     void* q_hat, const mla_decode_opts_t* opts, mla_stream_t stream);

/* a3+a4: scores s_j = softmax_scale * (q_hat . cache_row_j) over keys
 * 0..m, softmax, o_lat = sum_j p_j c_KV,j.  o_lat [B][q_len][H][d_c]. */
int mla_attend_latent(const mla_dims_t* dims, const void* q_hat, const mla_cache_t* cache,
                      const int32_t* seqlens, int32_t B, int32_t q_len, void* o_lat,
                      void* workspace, size_t workspace_bytes,
                      const mla_decode_opts_t* opts, mla_stream_t stream);

/* a5: out[r][h] = W_UV[h] o_lat[r][h] for the `rows` = B*q_len query tokens. */
int mla_project_out(const mla_dims_t* dims, const void* o_lat, const void* W_UV,
                    int32_t rows, void* out, const mla_decode_opts_t* opts,
                    mla_stream_t stream);

/* ---------------------------------------------------------------- projections around the decode
 * Both are dense bf16 contractions on the tensor cores (split over K so that
 * a few hundred tokens still spread the weight read over every SM); both
 * need bf16, the V3 head geometry (d_c 512, d_r 64, H 128, d_v 128) and a
 * compute-capability 10.0 device (MLA_ERR_UNSUPPORTED otherwise), and
 * d_model a multiple of 64.  Each takes a workspace (fp32 split partials)
 * of the size its *_workspace_bytes() returns, 16-byte aligned, owned by
 * the call until the stream reaches its end.
 *
 * Cache append from the attention block's input (a1 with the projections
 * that produce its inputs fused in):
 *   row pos[b]+i of sequence b = [ RMSNorm_gamma(W_DKV x[b][i]) || RoPE(W_KR x[b][i], pos[b]+i) ]
 * (m.lsln.cn/news/222502 section 2.2: c^KV = W^DKV h; section 1: RMSNorm,
 *  rms_norm_eps 1e-6 in its configuration block; 092 page, section 二: the
 *  cache keeps the latent and the decoupled RoPE key;
 *  ailearn.mscapital.top MLA panel: the hidden state is projected to c_KV
 *  and k_R).  The RMSNorm is taken over the d_c latent values in fp32.
 *   x      [B][n_tok][d_model]   block input (after the block's own pre-norm)
 *   W_A    [d_c + d_r][d_model]  rows 0..d_c-1 hold W_DKV, rows d_c.. hold W_KR
 *   gamma  [d_c]                 RMSNorm gain of the latent
 *   pos    [B] int32             position of the first new token of sequence b
 * Rows with an out-of-range position are skipped and set MLA_STATUS_BAD_POS. */
size_t mla_append_from_hidden_workspace_bytes(const mla_dims_t* dims, int32_t B, int32_t n_tok, int32_t d_model);
int mla_append_from_hidden(const mla_dims_t* dims, const void* x, const void* W_A, const void* gamma,
                           const int32_t* pos, int32_t B, int32_t n_tok, int32_t d_model,
                           const mla_cache_t* cache, void* workspace, size_t workspace_bytes,
                           mla_stream_t stream);

/* Output projection of the attention block: y[r] = W_O out[r], where out[r]
 * is a decode output row viewed as H * d_v values (head-major)
 * (ailearn.mscapital.top MLA panel: aggregate in latent space, then W_UV and
 * the output projection; taojin168.com forum page, section 2.1, the MLA
 * steps' last step: an output projection maps the attention output back to
 * the model width).
 *   attn_out [rows][H * d_v]     e.g. mla_decode's out, [B * q_len][H][d_v]
 *   W_O      [d_model][H * d_v]
 *   y        [rows][d_model]     written */
size_t mla_output_projection_workspace_bytes(const mla_dims_t* dims, int32_t rows, int32_t d_model);
int mla_output_projection(const mla_dims_t* dims, const void* attn_out, const void* W_O, int32_t rows,
                          int32_t d_model, void* y, void* workspace, size_t workspace_bytes,
                          mla_stream_t stream);

/* ---------------------------------------------------------------- status */

/* Synchronises `stream`, returns the device status word in *status (bits
 * MLA_STATUS_*) and clears it.  Returns MLA_OK, MLA_ERR_CUDA, or
 * MLA_ERR_DEVICE when the word was non-zero. */
int mla_device_status(mla_stream_t stream, int32_t* status);

/* Description of the last error on this host thread ("" if none). */
const char* mla_last_error(void);

/* Name of the path the last mla_decode* / step call on this thread used:
 * "sm100" or "generic". */
const char* mla_last_path(void);

/* ABI version (major*100 + minor). */
int mla_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MLA_H_ */
