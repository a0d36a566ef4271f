// Host launchers of the sm_100a path (bf16 storage, V3 head geometry:
// H = 128, d_c = 512, d_r = 64, d_n = 128, d_v = 128).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <string.h>

#include <utility>

#include "mla_internal.h"
#include "mla_rope.cuh"
#include "sm100_host.h"
#include "sm100_attend.cuh"
#include "sm100_gemm.cuh"
#include "sm100_gemv.cuh"

#ifdef MLA_TRACE
// Copies the attention kernel's timing trace (4096 tiles x 16 stamps) to host
// memory; only in builds compiled with -DMLA_TRACE.
extern "C" int mla_trace_read(void* host, size_t bytes) {
    return cudaMemcpyFromSymbol(host, mla::sm100::g_mla_trace, bytes) == cudaSuccess ? 0 : -4;
}
extern "C" int mla_trace_read_all(void* host, size_t bytes) {
    return cudaMemcpyFromSymbol(host, mla::sm100::g_mla_trace_all, bytes) == cudaSuccess ? 0 : -4;
}
extern "C" int mla_trace_read_kt(void* host, size_t bytes) {
    return cudaMemcpyFromSymbol(host, mla::sm100::g_mla_ktrace, bytes) == cudaSuccess ? 0 : -4;
}
extern "C" int mla_trace_clear_kt(void) {
    unsigned long long init[mla::sm100::kKtN][3];
    for (int k = 0; k < mla::sm100::kKtN; ++k) {
        init[k][0] = init[k][1] = ~0ull;
        init[k][2] = 0;
    }
    return cudaMemcpyToSymbol(mla::sm100::g_mla_ktrace, init, sizeof(init)) == cudaSuccess ? 0 : -4;
}
extern "C" int mla_trace_clear(void) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, mla::sm100::g_mla_trace) != cudaSuccess) return -4;
    if (cudaMemset(p, 0, sizeof(mla::sm100::g_mla_trace)) != cudaSuccess) return -4;
    if (cudaGetSymbolAddress(&p, mla::sm100::g_mla_trace_all) != cudaSuccess) return -4;
    return cudaMemset(p, 0, sizeof(mla::sm100::g_mla_trace_all)) == cudaSuccess ? 0 : -4;
}
#endif

namespace mla {

using namespace sm100;

namespace {

// ------------------------------------------------------------------ append

// One warp per new token: 16-byte copies of the 512 latent values and the
// RoPE rotation of the 64-wide key at its position (one pair per lane).
__global__ void append_v3_kernel(const __nv_bfloat16* __restrict__ c_kv, const __nv_bfloat16* __restrict__ k_rope,
                                 const int32_t* __restrict__ pos, int B, int n_tok, CacheView cache, RopeTable rope,
                                 int* status) {
    MLA_KT(kKtAppend, 0);
    const int gw = (blockIdx.x * blockDim.x + threadIdx.x) / 32;
    const int lane = threadIdx.x & 31;
    if (gw >= B * n_tok) return;
    const int b = gw / n_tok, i = gw % n_tok;
    const int p0 = pos[b];
    if (p0 < 0 || p0 + n_tok > cache.T_max) {
        if (lane == 0 && i == 0) atomicOr(status, MLA_STATUS_BAD_POS);
        return;
    }
    const int t = p0 + i;
    __nv_bfloat16* row = static_cast<__nv_bfloat16*>(cache.data) + (size_t)b * cache.stride_b + (size_t)t * cache.stride_t;
    const uint4* src = reinterpret_cast<const uint4*>(c_kv + (size_t)gw * kLat);
    uint4* dst = reinterpret_cast<uint4*>(row);
    dst[lane] = src[lane];
    dst[lane + 32] = src[lane + 32];
    const __nv_bfloat162 k2 = reinterpret_cast<const __nv_bfloat162*>(k_rope + (size_t)gw * kRope)[lane];
    float y0, y1;
    mla_rope_rotate(__low2float(k2), __high2float(k2), rope.inv_freq[lane], t, &y0, &y1);
    reinterpret_cast<__nv_bfloat162*>(row + kLat)[lane] = __floats2bfloat162_rn(y0, y1);
    MLA_KT(kKtAppend, 2);
}

bool g_smem_absorb[kMaxDev], g_smem_project[kMaxDev], g_smem_attend[kMaxDev];
bool g_smem_absorb_gemv[4][kMaxDev], g_smem_project_gemv[4][kMaxDev];

constexpr int kAbsorbStages = 2;
// Rows of the A tile a GEMM CTA loads: all 128 when the batch fills them,
// else the batch rounded up to 16 (the MMA still computes 128 rows; the rows
// past the batch are never stored).
int plan_ovh(int overhead_tiles) { return overhead_tiles < 0 ? 2 : overhead_tiles; }
int plan_min_units(int min_tiles) { return min_tiles > 0 ? min_tiles : 2; }
int gemm_a_rows(int rows) { return rows >= 128 ? 128 : ((rows + 15) / 16) * 16; }
constexpr int kProjStages = 4;
constexpr int kProjNT = 64;

}  // namespace

bool sm100_supported(const Problem& p, int q_len) {
    if (p.dtype != MLA_DTYPE_BF16 || p.H != kHeads || p.d_c != kLat || p.d_r != kRope || p.d_n != 128 ||
        p.d_v != 128)
        return false;
    if (q_len < 1 || q_len > 16) return false;
    int dev = 0, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    return major == 10 && minor == 0;
}

int sm100_default_pairs() { return device_sm_count() / 2; }

cudaError_t sm100_append(const Problem& p, const void* c_kv, const void* k_rope, const int32_t* pos, int n_tok,
                         const CacheView& cache, int* status, cudaStream_t st) {
    const int warps = p.B * n_tok;
    const int threads = 128;
    const int blocks = (warps * 32 + threads - 1) / threads;
    append_v3_kernel<<<blocks, threads, 0, st>>>((const __nv_bfloat16*)c_kv, (const __nv_bfloat16*)k_rope, pos, p.B,
                                                 n_tok, cache, p.rope, status);
    return cudaGetLastError();
}

cudaError_t sm100_absorb(const Problem& p, const void* q_nope, const void* q_rope, const void* W_UK,
                         const int32_t* seqlens, void* q_hat, cudaStream_t st, const PlanRequest* plan) {
    const int rows = p.B * p.q_len;
    CUtensorMap mA, mB;
    // A: q_nope viewed as [rows][H][128]; box 64 x 1 x 128 rows.
    if (!make_map(&mA, q_nope, 128, kHeads, rows, 128 * 2, (uint64_t)kHeads * 128 * 2, 64, 1, gemm_a_rows(rows),
                  CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    // B: W_UK viewed as [H][128 (d)][512 (c)]; box 64 c x 64 d x 1.
    if (!make_map(&mB, W_UK, kLat, 128, kHeads, kLat * 2, (uint64_t)128 * kLat * 2, 64, 64, 1,
                  CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    using Cfg = GemmCfg<2, 256, true, kAbsorbStages, true>;
    auto kern = head_gemm_kernel<2, 256, true, kAbsorbStages, true>;
    cudaError_t e = set_smem(kern, Cfg::kSmem, g_smem_absorb);
    if (e != cudaSuccess) return e;
    GemmArgs a;
    a.rows = rows;
    a.H = kHeads;
    a.ld_out = kRow;
    a.out_col0 = 0;
    a.out = (__nv_bfloat16*)q_hat;
    a.out_v8 = (reinterpret_cast<uintptr_t>(q_hat) & 31u) == 0;
    a.q_rope = (const __nv_bfloat16*)q_rope;
    a.seqlens = seqlens;
    a.q_len = p.q_len;
    a.rope = p.rope;
    a.status = device_status_ptr();
    a.a_rows = gemm_a_rows(rows);
    a.plan = nullptr;
    if (plan) {
        a.plan = static_cast<Plan*>(plan->plan);
        a.plan_B = p.B;
        a.plan_T_max = plan->T_max;
        a.plan_clusters = plan->clusters;
        a.plan_ovh = plan_ovh(plan->overhead_tiles);
        a.plan_min_units = plan_min_units(plan->min_tiles);
        a.plan_olat = static_cast<__nv_bfloat16*>(plan->o_lat);
    }
    dim3 grid(kHeads, kLat / 256, (rows + 127) / 128);
    return launch_pdl(kern, grid, dim3(128), Cfg::kSmem, st, 1, mA, mB, a);
}

cudaError_t sm100_project(const Problem& p, const void* o_lat, const void* W_UV, int rows, void* out,
                          cudaStream_t st) {
    CUtensorMap mA, mB;
    // A: o_lat viewed as [rows][H][512]; box 64 x 1 x 128.
    if (!make_map(&mA, o_lat, kLat, kHeads, rows, kLat * 2, (uint64_t)kHeads * kLat * 2, 64, 1, gemm_a_rows(rows),
                  CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    // B: W_UV viewed as [H][128 (d)][512 (c)]; box 64 c x NT d x 1 (K-major).
    if (!make_map(&mB, W_UV, kLat, 128, kHeads, kLat * 2, (uint64_t)128 * kLat * 2, 64, kProjNT, 1,
                  CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    using Cfg = GemmCfg<8, kProjNT, false, kProjStages, false>;
    auto kern = head_gemm_kernel<8, kProjNT, false, kProjStages, false>;
    cudaError_t e = set_smem(kern, Cfg::kSmem, g_smem_project);
    if (e != cudaSuccess) return e;
    GemmArgs a;
    memset(&a, 0, sizeof(a));
    a.plan = nullptr;
    a.rows = rows;
    a.H = kHeads;
    a.ld_out = 128;
    a.out_col0 = 0;
    a.out = (__nv_bfloat16*)out;
    a.out_v8 = (reinterpret_cast<uintptr_t>(out) & 31u) == 0;
    a.status = device_status_ptr();
    a.q_len = 1;
    a.a_rows = gemm_a_rows(rows);
    dim3 grid(kHeads, 128 / kProjNT, (rows + 127) / 128);
    return launch_pdl(kern, grid, dim3(128), Cfg::kSmem, st, 1, mA, mB, a);
}

// Small batches (rows <= kGemvMaxRows): CUDA-core matrix-vector kernels with
// the weight slices staged in shared memory; R = rows rounded up to 1, 2, 4, 8.
template <int R>
static cudaError_t absorb_gemv_launch(const AbsorbGemvArgs& a, cudaStream_t st) {
    static_assert(R == 1 || R == 2 || R == 4 || R == 8, "row count");
    constexpr int idx = R == 1 ? 0 : R == 2 ? 1 : R == 4 ? 2 : 3;
    cudaError_t e = set_smem(absorb_gemv_kernel<R>, absorb_gemv_smem<R>(), g_smem_absorb_gemv[idx]);
    if (e != cudaSuccess) return e;
    // W_UK [128 heads][128][512]: one box of 256 latent columns x 128 rows per CTA
    CUtensorMap mapW;
    if (!make_map(&mapW, a.W_UK, kLat, 128, kHeads, (uint64_t)kLat * 2, (uint64_t)128 * kLat * 2, 256, 128, 1,
                  CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    return launch_pdl(absorb_gemv_kernel<R>, dim3(kHeads + 1, 2), dim3(128), absorb_gemv_smem<R>(), st, 1, mapW, a);
}
template <int R>
static cudaError_t project_gemv_launch(const ProjectGemvArgs& a, cudaStream_t st) {
    constexpr int idx = R == 1 ? 0 : R == 2 ? 1 : R == 4 ? 2 : 3;
    cudaError_t e = set_smem(project_gemv_kernel<R>, project_gemv_smem<R>(), g_smem_project_gemv[idx]);
    if (e != cudaSuccess) return e;
    // W_UV [128 heads][128][512]: eight SW128 boxes of 64 latent columns x 128 rows per CTA
    CUtensorMap mapW;
    if (!make_map(&mapW, a.W_UV, kLat, 128, kHeads, (uint64_t)kLat * 2, (uint64_t)128 * kLat * 2, 64, 128, 1,
                  CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    return launch_pdl(project_gemv_kernel<R>, dim3(kHeads), dim3(512), project_gemv_smem<R>(), st, 1, mapW, a);
}

cudaError_t sm100_absorb_small(const Problem& p, const void* q_nope, const void* q_rope, const void* W_UK,
                               const int32_t* seqlens, void* q_hat, cudaStream_t st, const PlanRequest* plan) {
    const int rows = p.B * p.q_len;
    if (rows < 1 || rows > kGemvMaxRows) return cudaErrorInvalidValue;
    AbsorbGemvArgs a;
    memset(&a, 0, sizeof(a));
    a.q_nope = (const __nv_bfloat16*)q_nope;
    a.q_rope = (const __nv_bfloat16*)q_rope;
    a.W_UK = (const __nv_bfloat16*)W_UK;
    a.seqlens = seqlens;
    a.rows = rows;
    a.q_len = p.q_len;
    a.q_hat = (__nv_bfloat16*)q_hat;
    a.rope = p.rope;
    a.status = device_status_ptr();
    a.plan = nullptr;
    if (plan) {
        a.plan = static_cast<Plan*>(plan->plan);
        a.plan_B = p.B;
        a.plan_T_max = plan->T_max;
        a.plan_clusters = plan->clusters;
        a.plan_ovh = plan_ovh(plan->overhead_tiles);
        a.plan_min_units = plan_min_units(plan->min_tiles);
        a.plan_olat = static_cast<__nv_bfloat16*>(plan->o_lat);
    }
    if (rows == 1) return absorb_gemv_launch<1>(a, st);
    if (rows == 2) return absorb_gemv_launch<2>(a, st);
    if (rows <= 4) return absorb_gemv_launch<4>(a, st);
    return absorb_gemv_launch<8>(a, st);
}

// Clusters of the attention grid: at least one per query token (a group of
// q_len clusters streams one sequence piece, one cluster per token).
static int attend_clusters(int pairs, int q_len) { return pairs < q_len ? q_len : pairs; }

// Workspace of the attention step: plan, fp32 partials and LSEs.
static size_t attend_layout(const Problem& p, int pairs, size_t* off_part, size_t* off_lse) {
    const int clusters = attend_clusters(pairs, p.q_len);
    Carve c(nullptr);
    const size_t units = (size_t)p.B * p.q_len;  // one per query token
    c.take(sizeof(Plan) + sizeof(int) * (kPlanMaxGroups + 2 * units + 1));
    const size_t slots = (size_t)clusters + units;
    *off_part = c.off;
    c.take(slots * kHeads * kLat * sizeof(float));
    *off_lse = c.off;
    c.take(slots * kHeads * sizeof(float));
    return c.off;
}

void* sm100_plan_ptr(void* attend_workspace) { return attend_workspace; }

size_t sm100_attend_workspace_bytes(const Problem& p, int num_pairs) {
    size_t a, b;
    return attend_layout(p, num_pairs, &a, &b);
}

cudaError_t sm100_attend(const Problem& p, const void* q_hat, const CacheView& cache, const int32_t* seqlens,
                         void* o_lat, void* workspace, size_t ws_bytes, int num_pairs, int overhead_tiles,
                         int min_tiles, int* status, cudaStream_t st, const Events* events, bool plan_ready,
                         bool combine, const void* prefetch, size_t prefetch_bytes, const mla_decode_opts_t* opts) {
    const int clusters = attend_clusters(num_pairs, p.q_len);
    if (clusters / p.q_len > kPlanMaxGroups) return cudaErrorInvalidValue;
    size_t off_part, off_lse;
    const size_t need = attend_layout(p, clusters, &off_part, &off_lse);
    if (ws_bytes < need) return cudaErrorInvalidValue;
    char* ws = static_cast<char*>(workspace);
    Plan* plan = reinterpret_cast<Plan*>(ws);
    // The cache as [B][T_max][576]: boxes of 64 columns x 64 keys (SW128); the
    // scoring CTA loads all nine of a row tile, the accumulating CTA the eight
    // latent ones.
    CUtensorMap mRow;
    const uint64_t sb = (uint64_t)cache.stride_b * 2, stt = (uint64_t)cache.stride_t * 2;
    if (!make_map(&mRow, cache.data, kRow, cache.T_max, p.B, stt, sb, 64, kNk, 1, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;

    cudaError_t e;
    if (!plan_ready) {
        mla_plan_kernel<<<1, 32, 0, st>>>(seqlens, p.B, p.q_len, cache.T_max, clusters, plan_ovh(overhead_tiles),
                                          plan_min_units(min_tiles), plan, status, (__nv_bfloat16*)o_lat);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }

    e = set_smem(mla_attend_kernel, kAttSmem, g_smem_attend);
    if (e != cudaSuccess) return e;
    AttendArgs a;
    a.plan = plan;
    a.seqlens = seqlens;
    a.q_len = p.q_len;
    a.scale_log2 = p.scale * 1.4426950408889634f;
    a.q_hat = (const __nv_bfloat16*)q_hat;
    a.o_lat = (__nv_bfloat16*)o_lat;
    a.o_lat_v8 = (reinterpret_cast<uintptr_t>(o_lat) & 31u) == 0;
    a.prefetch = static_cast<const uint8_t*>(prefetch);
    a.prefetch_bytes = prefetch ? prefetch_bytes : 0;
    a.part_o = reinterpret_cast<float*>(ws + off_part);
    a.part_lse = reinterpret_cast<float*>(ws + off_lse);
    a.status = status;
    a.wait_limit_ns = (opts && opts->wait_limit_ns > 0) ? (uint64_t)opts->wait_limit_ns : MLA_WAIT_LIMIT_NS;
    a.withhold_tile = (opts && opts->withhold_tile > 0) ? opts->withhold_tile : -1;
    a.cache = static_cast<const uint8_t*>(cache.data);
    a.stride_b = cache.stride_b * 2;
    a.stride_t = cache.stride_t * 2;
    a.T_max = cache.T_max;

    if (events) events->record(MLA_EV_ATTEND_BEGIN, st);
    e = launch_pdl(mla_attend_kernel, dim3(clusters * 2), dim3(kAttThreads), kAttSmem, st, 2, mRow, a);
    if (e != cudaSuccess) return e;
    if (events) events->record(MLA_EV_ATTEND_END, st);

    // Split units number at most min(B * q_len, clusters); one CTA covers
    // eight heads of one unit.
    const int units = p.B * p.q_len;
    const int max_split = units < clusters ? units : clusters;
    if (combine)
        e = launch_pdl(mla_combine_kernel, dim3(max_split * (kHeads / 8)), dim3(256), 0, st, 1, (const Plan*)plan,
                       (const float*)a.part_o, (const float*)a.part_lse, (__nv_bfloat16*)o_lat);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t sm100_project_small(const Problem& p, void* attend_workspace, int num_pairs, const void* o_lat,
                                const void* W_UV, void* out, cudaStream_t st) {
    const int rows = p.B * p.q_len;
    if (rows < 1 || rows > kGemvMaxRows) return cudaErrorInvalidValue;
    size_t off_part, off_lse;
    attend_layout(p, num_pairs, &off_part, &off_lse);
    char* ws = static_cast<char*>(attend_workspace);
    ProjectGemvArgs a;
    a.plan = reinterpret_cast<const Plan*>(ws);
    a.o_lat = (const __nv_bfloat16*)o_lat;
    a.part_o = reinterpret_cast<const float*>(ws + off_part);
    a.part_lse = reinterpret_cast<const float*>(ws + off_lse);
    a.W_UV = (const __nv_bfloat16*)W_UV;
    a.rows = rows;
    a.out = (__nv_bfloat16*)out;
    a.status = device_status_ptr();
    if (rows == 1) return project_gemv_launch<1>(a, st);
    if (rows == 2) return project_gemv_launch<2>(a, st);
    if (rows <= 4) return project_gemv_launch<4>(a, st);
    return project_gemv_launch<8>(a, st);
}

}  // namespace mla
