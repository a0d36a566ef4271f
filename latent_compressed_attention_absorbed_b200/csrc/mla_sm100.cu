// Host launchers of the sm_100a path (bf16 storage, V3 head geometry:
// H = 128, d_c = 512, d_r = 64, d_n = 128, d_v = 128).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <string.h>

#include "mla_internal.h"
#include "mla_rope.cuh"
#include "sm100_attend.cuh"
#include "sm100_gemm.cuh"

#ifdef MLA_TRACE
// Copies the attention kernel's timing trace (4096 tiles x 16 stamps) to host
// memory; only in builds compiled with -DMLA_TRACE.
extern "C" int mla_trace_read(void* host, size_t bytes) {
    return cudaMemcpyFromSymbol(host, mla::sm100::g_mla_trace, bytes) == cudaSuccess ? 0 : -4;
}
#endif

namespace mla {

using namespace sm100;

namespace {

// ------------------------------------------------------------------ tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 3-D bf16 map: dims (d0 innermost, d1, d2), byte strides of d1 and d2, box (b0, b1, b2).
bool make_map(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1, uint64_t s2,
              uint32_t b0, uint32_t b1, uint32_t b2, CUtensorMapSwizzle sw) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {d0, d1, d2};
    const cuuint64_t strides[2] = {s1, s2};
    const cuuint32_t box[3] = {b0, b1, b2};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ append

// One warp per new token: 16-byte copies of the 512 latent values and the
// RoPE rotation of the 64-wide key at its position (one pair per lane).
__global__ void append_v3_kernel(const __nv_bfloat16* __restrict__ c_kv, const __nv_bfloat16* __restrict__ k_rope,
                                 const int32_t* __restrict__ pos, int B, int n_tok, CacheView cache, float base,
                                 int* status) {
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
    mla_rope_pair(__low2float(k2), __high2float(k2), lane, kRope, t, base, &y0, &y1);
    reinterpret_cast<__nv_bfloat162*>(row + kLat)[lane] = __floats2bfloat162_rn(y0, y1);
}

// Opt a kernel into more than 48 KB of dynamic shared memory, once per device
// and call site (`done` is that site's own flag array), so that later calls,
// including ones under stream capture, make no attribute calls.
constexpr int kMaxDev = 64;
template <typename K>
cudaError_t set_smem(K kernel, int bytes, bool (&done)[kMaxDev]) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < kMaxDev && done[dev]) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && dev >= 0 && dev < kMaxDev) done[dev] = true;
    return e;
}
bool g_smem_absorb[kMaxDev], g_smem_project[kMaxDev], g_smem_attend[kMaxDev];

constexpr int kAbsorbStages = 2;
constexpr int kProjStages = 4;
constexpr int kProjNT = 64;

}  // namespace

bool sm100_supported(const Problem& p, int q_len) {
    if (p.dtype != MLA_DTYPE_BF16 || p.H != kHeads || p.d_c != kLat || p.d_r != kRope || p.d_n != 128 ||
        p.d_v != 128)
        return false;
    if (q_len < 1 || q_len > 4) return false;
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
                                                 n_tok, cache, p.rope_base, status);
    return cudaGetLastError();
}

cudaError_t sm100_absorb(const Problem& p, const void* q_nope, const void* q_rope, const void* W_UK,
                         const int32_t* seqlens, void* q_hat, cudaStream_t st) {
    const int rows = p.B * p.q_len;
    CUtensorMap mA, mB;
    // A: q_nope viewed as [rows][H][128]; box 64 x 1 x 128 rows.
    if (!make_map(&mA, q_nope, 128, kHeads, rows, 128 * 2, (uint64_t)kHeads * 128 * 2, 64, 1, 128,
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
    a.q_rope = (const __nv_bfloat16*)q_rope;
    a.seqlens = seqlens;
    a.q_len = p.q_len;
    a.rope_base = p.rope_base;
    a.status = device_status_ptr();
    dim3 grid(kHeads, kLat / 256, (rows + 127) / 128);
    kern<<<grid, 128, Cfg::kSmem, st>>>(mA, mB, a);
    return cudaGetLastError();
}

cudaError_t sm100_project(const Problem& p, const void* o_lat, const void* W_UV, int rows, void* out,
                          cudaStream_t st) {
    CUtensorMap mA, mB;
    // A: o_lat viewed as [rows][H][512]; box 64 x 1 x 128.
    if (!make_map(&mA, o_lat, kLat, kHeads, rows, kLat * 2, (uint64_t)kHeads * kLat * 2, 64, 1, 128,
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
    a.rows = rows;
    a.H = kHeads;
    a.ld_out = 128;
    a.out_col0 = 0;
    a.out = (__nv_bfloat16*)out;
    a.status = device_status_ptr();
    a.q_len = 1;
    dim3 grid(kHeads, 128 / kProjNT, (rows + 127) / 128);
    kern<<<grid, 128, Cfg::kSmem, st>>>(mA, mB, a);
    return cudaGetLastError();
}

// Workspace of the attention step: plan, fp32 partials and LSEs.
static size_t attend_layout(const Problem& p, int clusters, size_t* off_part, size_t* off_lse) {
    Carve c(nullptr);
    c.take(sizeof(Plan) + sizeof(int) * (p.B + 1));
    const size_t slots = (size_t)clusters + p.B;
    *off_part = c.off;
    c.take(slots * p.q_len * kHeads * kLat * sizeof(float));
    *off_lse = c.off;
    c.take(slots * p.q_len * kHeads * sizeof(float));
    return c.off;
}

size_t sm100_attend_workspace_bytes(const Problem& p, int num_pairs) {
    size_t a, b;
    return attend_layout(p, num_pairs, &a, &b);
}

cudaError_t sm100_attend(const Problem& p, const void* q_hat, const CacheView& cache, const int32_t* seqlens,
                         void* o_lat, void* workspace, size_t ws_bytes, int num_pairs, int overhead_tiles,
                         int* status, cudaStream_t st, const Events* events) {
    const int clusters = num_pairs;
    size_t off_part, off_lse;
    const size_t need = attend_layout(p, clusters, &off_part, &off_lse);
    if (ws_bytes < need) return cudaErrorInvalidValue;
    char* ws = static_cast<char*>(workspace);
    Plan* plan = reinterpret_cast<Plan*>(ws);
    CUtensorMap mC;
    const uint64_t sb = (uint64_t)cache.stride_b * 2, stt = (uint64_t)cache.stride_t * 2;
    if (!make_map(&mC, cache.data, kRow, cache.T_max, p.B, stt, sb, 64, kNk, 1, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;

    const int ovh = overhead_tiles < 0 ? 2 : overhead_tiles;
    mla_plan_kernel<<<1, 1024, 0, st>>>(seqlens, p.B, p.q_len, cache.T_max, clusters, ovh, 1, plan, status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    e = set_smem(mla_attend_kernel, kAttSmem, g_smem_attend);
    if (e != cudaSuccess) return e;
    AttendArgs a;
    a.plan = plan;
    a.seqlens = seqlens;
    a.q_len = p.q_len;
    a.T_max = cache.T_max;
    a.scale_log2 = p.scale * 1.4426950408889634f;
    a.q_hat = (const __nv_bfloat16*)q_hat;
    a.o_lat = (__nv_bfloat16*)o_lat;
    a.part_o = reinterpret_cast<float*>(ws + off_part);
    a.part_lse = reinterpret_cast<float*>(ws + off_lse);
    a.status = status;

    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    const int csize = 2 * p.q_len;
    cfg.gridDim = dim3(clusters * csize, 1, 1);
    cfg.blockDim = dim3(kAttThreads, 1, 1);
    cfg.dynamicSmemBytes = kAttSmem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = csize;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (events) events->record(MLA_EV_ATTEND_BEGIN, st);
    e = cudaLaunchKernelEx(&cfg, mla_attend_kernel, mC, a);
    if (e != cudaSuccess) return e;
    if (events) events->record(MLA_EV_ATTEND_END, st);

    const int warps = p.B * p.q_len * kHeads;
    mla_combine_kernel<<<(warps * 32 + 255) / 256, 256, 0, st>>>(plan, a.part_o, a.part_lse, p.q_len,
                                                                 (__nv_bfloat16*)o_lat);
    return cudaGetLastError();
}

}  // namespace mla
