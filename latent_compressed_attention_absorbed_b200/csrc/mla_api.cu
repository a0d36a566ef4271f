// C ABI of libmla.so (declared in include/mla.h): argument checks, path
// selection, workspace carving and the device status word.
#include <cuda_runtime.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "mla_internal.h"

namespace mla {

// Bits of MLA_STATUS_* raised by kernels of this library on this device.
static __device__ int g_status_word;

namespace {

thread_local char t_err[512] = "";
thread_local const char* t_path = "";

int fail(int code, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(t_err, sizeof(t_err), fmt, ap);
    va_end(ap);
    return code;
}

int cuda_fail(cudaError_t e, const char* what) {
    return fail(MLA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int* g_status_ptr[kMaxDevices];
int g_sm_count[kMaxDevices];

int current_device() {
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess) return -1;
    return d;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

int check_dims(const mla_dims_t* d, Problem* p) {
    if (!d) return fail(MLA_ERR_ARG, "dims is NULL");
    if (d->H <= 0 || d->d_c <= 0 || d->d_r < 0 || d->d_n <= 0 || d->d_v <= 0)
        return fail(MLA_ERR_SHAPE, "head dimensions must be positive (H=%d d_c=%d d_r=%d d_n=%d d_v=%d)", d->H,
                    d->d_c, d->d_r, d->d_n, d->d_v);
    if (d->d_r % 2) return fail(MLA_ERR_SHAPE, "d_r must be even (RoPE pairs), got %d", d->d_r);
    if (d->d_r > 128) return fail(MLA_ERR_SHAPE, "d_r > 128 is not supported");
    if (d->d_c > 1024) return fail(MLA_ERR_SHAPE, "d_c > 1024 is not supported");
    if (d->dtype != MLA_DTYPE_BF16 && d->dtype != MLA_DTYPE_F32) return fail(MLA_ERR_ARG, "unknown dtype %d", d->dtype);
    if (!(d->rope_base > 0.f)) return fail(MLA_ERR_ARG, "rope_base must be > 0");
    if (d->softmax_scale < 0.f) return fail(MLA_ERR_ARG, "softmax_scale must be >= 0");
    p->H = d->H;
    p->d_c = d->d_c;
    p->d_r = d->d_r;
    p->d_n = d->d_n;
    p->d_v = d->d_v;
    p->dtype = d->dtype;
    p->rope_base = d->rope_base;
    p->scale = d->softmax_scale > 0.f ? d->softmax_scale : 1.0f / sqrtf((float)(d->d_n + d->d_r));
    p->B = 0;
    p->q_len = 1;
    for (int k = 0; k < 64; ++k)
        p->rope.inv_freq[k] = (k < d->d_r / 2) ? pow((double)d->rope_base, -2.0 * k / (double)d->d_r) : 0.0;
    return MLA_OK;
}

size_t elem_size(const Problem& p) { return p.dtype == MLA_DTYPE_F32 ? 4 : 2; }

int check_cache(const Problem& p, const mla_cache_t* c, int B, CacheView* v) {
    if (!c || !c->data) return fail(MLA_ERR_ARG, "cache or cache->data is NULL");
    if (!aligned16(c->data)) return fail(MLA_ERR_ALIGN, "cache->data must be 16-byte aligned");
    if (c->B < B) return fail(MLA_ERR_SHAPE, "cache holds %d sequences, call needs %d", c->B, B);
    if (c->T_max <= 0) return fail(MLA_ERR_SHAPE, "cache T_max must be positive");
    const int64_t row = p.d_c + p.d_r;
    if (c->stride_t < row) return fail(MLA_ERR_SHAPE, "cache stride_t %lld < row width %lld", (long long)c->stride_t,
                                       (long long)row);
    if (c->stride_b < c->stride_t * (int64_t)c->T_max && c->B > 1)
        return fail(MLA_ERR_SHAPE, "cache stride_b smaller than T_max * stride_t");
    const int64_t es = (int64_t)elem_size(p);
    if ((c->stride_t * es) % 16 || (c->stride_b * es) % 16)
        return fail(MLA_ERR_ALIGN, "cache strides must be multiples of 16 bytes");
    v->data = c->data;
    v->T_max = c->T_max;
    v->stride_b = c->stride_b;
    v->stride_t = c->stride_t;
    return MLA_OK;
}

int choose_path(const Problem& p, int q_len, const mla_decode_opts_t* o, bool* fast) {
    const int want = o ? o->path : 0;
    if (want < 0 || want > 2) return fail(MLA_ERR_ARG, "opts->path must be 0, 1 or 2");
    const bool can = sm100_supported(p, q_len);
    if (want == 1 && !can)
        return fail(MLA_ERR_UNSUPPORTED,
                    "the sm_100a path needs a compute-capability 10.0 device, bf16, H=128, d_c=512, d_r=64, "
                    "d_n=128, d_v=128 and q_len <= 16");
    *fast = (want == 1) || (want == 0 && can);
    t_path = *fast ? "sm100" : "generic";
    return MLA_OK;
}

int pairs_for(const mla_decode_opts_t* o) {
    // At most the clusters that fit on the device at once: more would only
    // run in a second wave, and mla_workspace_bytes() sizes for that many.
    const int cap = sm100_default_pairs();
    int n = (o && o->num_pairs > 0 && o->num_pairs < cap) ? o->num_pairs : cap;
    if (n > 1024) n = 1024;  // the split combine handles at most 1024 pieces per sequence
    return n > 0 ? n : 1;
}

// The kernels store 32-byte vectors into the workspace; its base is rounded up
// to 256 bytes inside the caller's buffer (mla_workspace_bytes includes the
// slack), so any 16-byte-aligned buffer of that size works.
constexpr size_t kWsAlign = 256;
void* align_ws(void* ws, size_t* bytes) {
    const uintptr_t p = reinterpret_cast<uintptr_t>(ws);
    const uintptr_t a = (p + kWsAlign - 1) & ~uintptr_t(kWsAlign - 1);
    *bytes = (a - p) > *bytes ? 0 : *bytes - (a - p);
    return reinterpret_cast<void*>(a);
}

struct DecodeLayout {
    size_t q_hat, o_lat, attend, total;
};

DecodeLayout decode_layout(const Problem& p, bool fast, int pairs) {
    Carve c(nullptr);
    DecodeLayout L;
    const size_t U = (size_t)p.B * p.q_len * p.H;
    L.q_hat = c.off;
    c.take(U * (p.d_c + p.d_r) * elem_size(p));
    L.o_lat = c.off;
    c.take(U * p.d_c * elem_size(p));
    L.attend = c.off;
    if (fast) c.take(sm100_attend_workspace_bytes(p, pairs));
    L.total = c.off;
    return L;
}

}  // namespace

int set_error(int code, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(t_err, sizeof(t_err), fmt, ap);
    va_end(ap);
    return code;
}

int* device_status_ptr() {
    const int d = current_device();
    if (d < 0 || d >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> g(g_mu);
    if (!g_status_ptr[d]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_status_word) != cudaSuccess) return nullptr;
        g_status_ptr[d] = static_cast<int*>(ptr);
    }
    return g_status_ptr[d];
}

int device_sm_count() {
    const int d = current_device();
    if (d < 0 || d >= kMaxDevices) return 1;
    std::lock_guard<std::mutex> g(g_mu);
    if (!g_sm_count[d]) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d);
        g_sm_count[d] = n > 0 ? n : 1;
    }
    return g_sm_count[d];
}

}  // namespace mla

using namespace mla;

extern "C" {

int mla_version(void) { return 101; }

const char* mla_last_error(void) { return t_err; }

const char* mla_last_path(void) { return t_path; }

int mla_append_cache(const mla_dims_t* dims, const void* c_kv, const void* k_rope, const int32_t* pos, int32_t B,
                     int32_t n_tok, const mla_cache_t* cache, mla_stream_t stream) {
    t_err[0] = 0;
    Problem p;
    int rc = check_dims(dims, &p);
    if (rc) return rc;
    if (B < 0 || n_tok < 0) return fail(MLA_ERR_ARG, "B and n_tok must be >= 0");
    if (B == 0 || n_tok == 0) return MLA_OK;
    if (!c_kv || !k_rope || !pos) return fail(MLA_ERR_ARG, "NULL tensor pointer");
    if (!aligned16(c_kv) || !aligned16(k_rope) || !aligned4(pos)) return fail(MLA_ERR_ALIGN, "misaligned pointer");
    CacheView cv;
    rc = check_cache(p, cache, B, &cv);
    if (rc) return rc;
    p.B = B;
    int* status = device_status_ptr();
    if (!status) return fail(MLA_ERR_CUDA, "no CUDA device / status word");
    const bool fast = sm100_supported(p, 1);
    t_path = fast ? "sm100" : "generic";
    cudaError_t e = fast ? sm100_append(p, c_kv, k_rope, pos, n_tok, cv, status, (cudaStream_t)stream)
                         : generic_append(p, c_kv, k_rope, pos, n_tok, cv, status, (cudaStream_t)stream);
    return e == cudaSuccess ? MLA_OK : cuda_fail(e, "append launch");
}

size_t mla_workspace_bytes(const mla_dims_t* dims, int32_t B, int32_t q_len) {
    Problem p;
    if (check_dims(dims, &p) || B < 0 || q_len < 1) return 0;
    p.B = B;
    p.q_len = q_len;
    const bool fast = sm100_supported(p, q_len);
    const DecodeLayout g = decode_layout(p, false, 1);
    if (!fast) return g.total + kWsAlign;
    const DecodeLayout f = decode_layout(p, true, sm100_default_pairs());
    return (f.total > g.total ? f.total : g.total) + kWsAlign;
}

int mla_absorb_query(const mla_dims_t* dims, const void* q_nope, const void* q_rope, const void* W_UK,
                     const int32_t* seqlens, int32_t B, int32_t q_len, void* q_hat, const mla_decode_opts_t* opts,
                     mla_stream_t stream) {
    t_err[0] = 0;
    Problem p;
    int rc = check_dims(dims, &p);
    if (rc) return rc;
    if (B < 0 || q_len < 1 || q_len > 16) return fail(MLA_ERR_ARG, "need B >= 0 and 1 <= q_len <= 16");
    if (B == 0) return MLA_OK;
    if (!q_nope || !q_rope || !W_UK || !seqlens || !q_hat) return fail(MLA_ERR_ARG, "NULL tensor pointer");
    if (!aligned16(q_nope) || !aligned16(q_rope) || !aligned16(W_UK) || !aligned16(q_hat) || !aligned4(seqlens))
        return fail(MLA_ERR_ALIGN, "misaligned pointer");
    p.B = B;
    p.q_len = q_len;
    bool fast;
    rc = choose_path(p, q_len, opts, &fast);
    if (rc) return rc;
    cudaError_t e = fast ? sm100_absorb(p, q_nope, q_rope, W_UK, seqlens, q_hat, (cudaStream_t)stream)
                         : generic_absorb(p, q_nope, q_rope, W_UK, seqlens, q_hat, (cudaStream_t)stream);
    return e == cudaSuccess ? MLA_OK : cuda_fail(e, "absorb launch");
}

int mla_attend_latent(const mla_dims_t* dims, const void* q_hat, const mla_cache_t* cache, const int32_t* seqlens,
                      int32_t B, int32_t q_len, void* o_lat, void* workspace, size_t workspace_bytes,
                      const mla_decode_opts_t* opts, mla_stream_t stream) {
    t_err[0] = 0;
    Problem p;
    int rc = check_dims(dims, &p);
    if (rc) return rc;
    if (B < 0 || q_len < 1 || q_len > 16) return fail(MLA_ERR_ARG, "need B >= 0 and 1 <= q_len <= 16");
    if (B == 0) return MLA_OK;
    if (!q_hat || !seqlens || !o_lat) return fail(MLA_ERR_ARG, "NULL tensor pointer");
    if (!aligned16(q_hat) || !aligned16(o_lat) || !aligned4(seqlens)) return fail(MLA_ERR_ALIGN, "misaligned pointer");
    CacheView cv;
    rc = check_cache(p, cache, B, &cv);
    if (rc) return rc;
    p.B = B;
    p.q_len = q_len;
    bool fast;
    rc = choose_path(p, q_len, opts, &fast);
    if (rc) return rc;
    int* status = device_status_ptr();
    if (!status) return fail(MLA_ERR_CUDA, "no CUDA device / status word");
    cudaError_t e;
    if (fast) {
        const int pairs = pairs_for(opts);
        const size_t need = sm100_attend_workspace_bytes(p, pairs) + kWsAlign;
        if (!workspace || workspace_bytes < need || !aligned16(workspace))
            return fail(MLA_ERR_WORKSPACE, "attend workspace needs %zu bytes (16-byte aligned), got %zu", need,
                        workspace_bytes);
        workspace = align_ws(workspace, &workspace_bytes);
        e = sm100_attend(p, q_hat, cv, seqlens, o_lat, workspace, workspace_bytes, pairs,
                         opts ? opts->overhead_tiles : -1, opts ? opts->min_tiles : 0, status, (cudaStream_t)stream,
                         nullptr, false, true, nullptr, 0, opts);
    } else {
        e = generic_attend(p, q_hat, cv, seqlens, o_lat, status, (cudaStream_t)stream);
    }
    return e == cudaSuccess ? MLA_OK : cuda_fail(e, "attend launch");
}

int mla_project_out(const mla_dims_t* dims, const void* o_lat, const void* W_UV, int32_t rows, void* out,
                    const mla_decode_opts_t* opts, mla_stream_t stream) {
    t_err[0] = 0;
    Problem p;
    int rc = check_dims(dims, &p);
    if (rc) return rc;
    if (rows < 0) return fail(MLA_ERR_ARG, "rows must be >= 0");
    if (rows == 0) return MLA_OK;
    if (!o_lat || !W_UV || !out) return fail(MLA_ERR_ARG, "NULL tensor pointer");
    if (!aligned16(o_lat) || !aligned16(W_UV) || !aligned16(out)) return fail(MLA_ERR_ALIGN, "misaligned pointer");
    p.B = rows;
    p.q_len = 1;
    bool fast;
    rc = choose_path(p, 1, opts, &fast);
    if (rc) return rc;
    cudaError_t e = fast ? sm100_project(p, o_lat, W_UV, rows, out, (cudaStream_t)stream)
                         : generic_project(p, o_lat, W_UV, rows, out, (cudaStream_t)stream);
    return e == cudaSuccess ? MLA_OK : cuda_fail(e, "project launch");
}

int mla_decode_ex(const mla_dims_t* dims, const void* q_nope, const void* q_rope, const void* W_UK, const void* W_UV,
                  const mla_cache_t* cache, const int32_t* seqlens, int32_t B, int32_t q_len, void* out,
                  void* workspace, size_t workspace_bytes, const mla_decode_opts_t* opts, mla_stream_t stream) {
    t_err[0] = 0;
    Problem p;
    int rc = check_dims(dims, &p);
    if (rc) return rc;
    if (B < 0 || q_len < 1 || q_len > 16) return fail(MLA_ERR_ARG, "need B >= 0 and 1 <= q_len <= 16");
    if (B == 0) return MLA_OK;
    if (!q_nope || !q_rope || !W_UK || !W_UV || !seqlens || !out) return fail(MLA_ERR_ARG, "NULL tensor pointer");
    if (!aligned16(q_nope) || !aligned16(q_rope) || !aligned16(W_UK) || !aligned16(W_UV) || !aligned16(out) ||
        !aligned4(seqlens))
        return fail(MLA_ERR_ALIGN, "misaligned pointer");
    CacheView cv;
    rc = check_cache(p, cache, B, &cv);
    if (rc) return rc;
    p.B = B;
    p.q_len = q_len;
    bool fast;
    rc = choose_path(p, q_len, opts, &fast);
    if (rc) return rc;
    const int pairs = fast ? pairs_for(opts) : 1;
    const DecodeLayout L = decode_layout(p, fast, pairs);
    if (!workspace || workspace_bytes < L.total + kWsAlign || !aligned16(workspace))
        return fail(MLA_ERR_WORKSPACE, "decode workspace needs %zu bytes (16-byte aligned), got %zu",
                    L.total + kWsAlign, workspace_bytes);
    workspace = align_ws(workspace, &workspace_bytes);
    int* status = device_status_ptr();
    if (!status) return fail(MLA_ERR_CUDA, "no CUDA device / status word");
    char* ws = static_cast<char*>(workspace);
    void* q_hat = ws + L.q_hat;
    void* o_lat = ws + L.o_lat;
    const cudaStream_t st = (cudaStream_t)stream;
    Events ev;
    if (opts && opts->events && opts->n_events >= MLA_NUM_EVENTS) {
        for (int i = 0; i < MLA_NUM_EVENTS; ++i) ev.ev[i] = (cudaEvent_t)opts->events[i];
        ev.on = true;
    }
    cudaError_t e;
    ev.record(MLA_EV_START, st);
    if (fast) {
        PlanRequest pr;
        pr.plan = ws + L.attend;
        pr.o_lat = o_lat;
        pr.T_max = cv.T_max;
        pr.clusters = pairs;
        pr.overhead_tiles = opts ? opts->overhead_tiles : -1;
        pr.min_tiles = opts ? opts->min_tiles : 0;
        const bool small = B * q_len <= kSmallRows;
        e = B * q_len <= kSmallAbsorbRows ? sm100_absorb_small(p, q_nope, q_rope, W_UK, seqlens, q_hat, st, &pr)
                                          : sm100_absorb(p, q_nope, q_rope, W_UK, seqlens, q_hat, st, &pr);
        ev.record(MLA_EV_ABSORB_DONE, st);
        // When the cache read is small the HBM idles during attention: prefetch
        // W_UV into L2 meanwhile (the cache bound is a cheap host-side bound:
        // B sequences of at most T_max rows).
        const size_t cache_bound = (size_t)B * cv.T_max * (p.d_c + p.d_r) * 2;
        const bool pf = cache_bound <= (size_t(64) << 20);
        if (e == cudaSuccess)
            e = sm100_attend(p, q_hat, cv, seqlens, o_lat, ws + L.attend, L.total - L.attend, pairs,
                             opts ? opts->overhead_tiles : -1, opts ? opts->min_tiles : 0, status, st, &ev,
                             /*plan_ready=*/true, /*combine=*/!small, pf ? W_UV : nullptr,
                             (size_t)p.H * p.d_v * p.d_c * 2, opts);
        ev.record(MLA_EV_COMBINE_DONE, st);
        if (e == cudaSuccess)
            e = small ? sm100_project_small(p, ws + L.attend, pairs, o_lat, W_UV, out, st)
                      : sm100_project(p, o_lat, W_UV, B * q_len, out, st);
    } else {
        e = generic_absorb(p, q_nope, q_rope, W_UK, seqlens, q_hat, st);
        ev.record(MLA_EV_ABSORB_DONE, st);
        if (e == cudaSuccess) e = generic_attend(p, q_hat, cv, seqlens, o_lat, status, st);
        ev.record(MLA_EV_ATTEND_BEGIN, st);
        ev.record(MLA_EV_ATTEND_END, st);
        ev.record(MLA_EV_COMBINE_DONE, st);
        if (e == cudaSuccess) e = generic_project(p, o_lat, W_UV, B * q_len, out, st);
    }
    ev.record(MLA_EV_END, st);
    t_path = fast ? "sm100" : "generic";
    return e == cudaSuccess ? MLA_OK : cuda_fail(e, "decode launch");
}

int mla_decode(const mla_dims_t* dims, const void* q_nope, const void* q_rope, const void* W_UK, const void* W_UV,
               const mla_cache_t* cache, const int32_t* seqlens, int32_t B, int32_t q_len, void* out, void* workspace,
               size_t workspace_bytes, mla_stream_t stream) {
    return mla_decode_ex(dims, q_nope, q_rope, W_UK, W_UV, cache, seqlens, B, q_len, out, workspace, workspace_bytes,
                         nullptr, stream);
}

size_t mla_append_from_hidden_workspace_bytes(const mla_dims_t* dims, int32_t B, int32_t n_tok, int32_t d_model) {
    Problem p;
    if (check_dims(dims, &p) || B < 0 || n_tok < 0 || d_model <= 0 || d_model % 64) return 0;
    return append_hidden_workspace(B * n_tok, d_model) + kWsAlign;
}

int mla_append_from_hidden(const mla_dims_t* dims, const void* x, const void* W_A, const void* gamma,
                           const int32_t* pos, int32_t B, int32_t n_tok, int32_t d_model, const mla_cache_t* cache,
                           void* workspace, size_t workspace_bytes, mla_stream_t stream) {
    t_err[0] = 0;
    Problem p;
    int rc = check_dims(dims, &p);
    if (rc) return rc;
    if (B < 0 || n_tok < 0 || d_model <= 0) return fail(MLA_ERR_ARG, "need B >= 0, n_tok >= 0, d_model > 0");
    if (d_model % 64) return fail(MLA_ERR_SHAPE, "d_model must be a multiple of 64, got %d", d_model);
    if (B == 0 || n_tok == 0) return MLA_OK;
    if (!x || !W_A || !gamma || !pos) return fail(MLA_ERR_ARG, "NULL tensor pointer");
    if (!aligned16(x) || !aligned16(W_A) || !aligned16(gamma) || !aligned4(pos))
        return fail(MLA_ERR_ALIGN, "misaligned pointer");
    p.B = B;
    if (!sm100_linear_supported(p))
        return fail(MLA_ERR_UNSUPPORTED,
                    "mla_append_from_hidden needs a compute-capability 10.0 device, bf16 and the V3 head geometry");
    CacheView cv;
    rc = check_cache(p, cache, B, &cv);
    if (rc) return rc;
    const size_t need = append_hidden_workspace(B * n_tok, d_model) + kWsAlign;
    if (!workspace || workspace_bytes < need || !aligned16(workspace))
        return fail(MLA_ERR_WORKSPACE, "append workspace needs %zu bytes (16-byte aligned), got %zu", need,
                    workspace_bytes);
    workspace = align_ws(workspace, &workspace_bytes);
    int* status = device_status_ptr();
    if (!status) return fail(MLA_ERR_CUDA, "no CUDA device / status word");
    t_path = "sm100";
    cudaError_t e = sm100_append_hidden(p, x, W_A, gamma, pos, n_tok, d_model, cv, workspace, status,
                                        (cudaStream_t)stream);
    return e == cudaSuccess ? MLA_OK : cuda_fail(e, "append-from-hidden launch");
}

size_t mla_output_projection_workspace_bytes(const mla_dims_t* dims, int32_t rows, int32_t d_model) {
    Problem p;
    if (check_dims(dims, &p) || rows < 0 || d_model <= 0 || d_model % 64) return 0;
    return output_projection_workspace(p, rows, d_model) + kWsAlign;
}

int mla_output_projection(const mla_dims_t* dims, const void* attn_out, const void* W_O, int32_t rows,
                          int32_t d_model, void* y, void* workspace, size_t workspace_bytes, mla_stream_t stream) {
    t_err[0] = 0;
    Problem p;
    int rc = check_dims(dims, &p);
    if (rc) return rc;
    if (rows < 0 || d_model <= 0) return fail(MLA_ERR_ARG, "need rows >= 0 and d_model > 0");
    if (d_model % 64) return fail(MLA_ERR_SHAPE, "d_model must be a multiple of 64, got %d", d_model);
    if (rows == 0) return MLA_OK;
    if (!attn_out || !W_O || !y) return fail(MLA_ERR_ARG, "NULL tensor pointer");
    if (!aligned16(attn_out) || !aligned16(W_O) || !aligned16(y)) return fail(MLA_ERR_ALIGN, "misaligned pointer");
    p.B = rows;
    if (!sm100_linear_supported(p))
        return fail(MLA_ERR_UNSUPPORTED,
                    "mla_output_projection needs a compute-capability 10.0 device, bf16 and the V3 head geometry");
    const size_t need = output_projection_workspace(p, rows, d_model) + kWsAlign;
    if (!workspace || workspace_bytes < need || !aligned16(workspace))
        return fail(MLA_ERR_WORKSPACE, "output-projection workspace needs %zu bytes (16-byte aligned), got %zu", need,
                    workspace_bytes);
    workspace = align_ws(workspace, &workspace_bytes);
    int* status = device_status_ptr();
    if (!status) return fail(MLA_ERR_CUDA, "no CUDA device / status word");
    t_path = "sm100";
    cudaError_t e = sm100_output_projection(p, attn_out, W_O, rows, d_model, y, workspace, status,
                                            (cudaStream_t)stream);
    return e == cudaSuccess ? MLA_OK : cuda_fail(e, "output-projection launch");
}

int mla_device_status(mla_stream_t stream, int32_t* status) {
    t_err[0] = 0;
    if (!status) return fail(MLA_ERR_ARG, "status is NULL");
    int* ptr = device_status_ptr();
    if (!ptr) return fail(MLA_ERR_CUDA, "no CUDA device / status word");
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
    int v = 0;
    e = cudaMemcpy(&v, ptr, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "status read");
    const int zero = 0;
    e = cudaMemcpy(ptr, &zero, sizeof(int), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "status clear");
    *status = v;
    if (v) return fail(MLA_ERR_DEVICE, "device status 0x%x", v);
    return MLA_OK;
}

}  // extern "C"
