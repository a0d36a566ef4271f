// The two dense projections around the attention step, and their C ABI:
//
//   mla_append_from_hidden: cache rows from the attention block's input x,
//       [ RMSNorm_gamma(W_DKV x) || RoPE(W_KR x, pos) ]
//       (m.lsln.cn/news/222502 section 2.2: c^KV = W^DKV h, and section 1:
//       RMSNorm in the V3 block; 092 page, section 二: the cache holds the
//       latent and the decoupled RoPE key; ailearn.mscapital.top MLA panel:
//       the hidden state is projected to c_KV and k_R);
//   mla_output_projection: y = W_O out, the per-head outputs of the decode
//       (H * d_v values per query token) mapped back to the hidden size
//       (ailearn.mscapital.top MLA panel: W_UV, then the output projection).
//
// Both run the split-K tcgen05 contraction of sm100_linear.cuh; a finishing
// kernel adds the split partials in a fixed order (bitwise reproducible)
// and applies the RMSNorm / RoPE epilogue (append) or rounds to bf16
// (output projection).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <string.h>

#include "mla_internal.h"
#include "mla_rope.cuh"
#include "sm100_host.h"
#include "sm100_linear.cuh"

namespace mla {

using namespace sm100;

namespace {

constexpr int kLat = 512;    // d_c
constexpr int kRope = 64;    // d_r
constexpr int kHeads = 128;  // H
constexpr int kLinNT = 64;
constexpr int kLinStages = 4;
using LinC = LinCfg<kLinNT, kLinStages>;
bool g_smem_linear[kMaxDev];
constexpr int kAppendRow = kLat + kRope;  // 576 outputs per token
constexpr float kRmsEps = 1e-6f;          // rms_norm_eps of the V3 configuration

// Splits of K: about two resident CTAs per SM over the (column tiles x row
// tiles) grid, at least four 64-wide K chunks per CTA.
int choose_splits(int tiles, int kc_total) {
    const int sms = device_sm_count();
    int s = (2 * sms) / (tiles > 0 ? tiles : 1);
    const int cap = kc_total / 4 > 0 ? kc_total / 4 : 1;
    if (s > cap) s = cap;
    return s > 0 ? s : 1;
}

struct LinPlan {
    int rows, N, K, kc_total, splits, kc_per_split, row_tiles, col_tiles;
};

LinPlan lin_plan(int rows, int N, int K) {
    LinPlan p;
    p.rows = rows;
    p.N = N;
    p.K = K;
    p.kc_total = K / 64;
    p.row_tiles = (rows + 127) / 128;
    p.col_tiles = N / kLinNT;
    p.splits = choose_splits(p.col_tiles * p.row_tiles, p.kc_total);
    p.kc_per_split = (p.kc_total + p.splits - 1) / p.splits;
    p.splits = (p.kc_total + p.kc_per_split - 1) / p.kc_per_split;  // no empty split
    return p;
}

size_t lin_partial_bytes(const LinPlan& p) { return p.splits > 1 ? (size_t)p.splits * p.rows * p.N * 4 : 0; }

int a_rows_for(int rows) { return rows >= 128 ? 128 : ((rows + 15) / 16) * 16; }

cudaError_t lin_launch(const LinPlan& p, const void* A, const void* B, float* part, __nv_bfloat16* out, int* status,
                       cudaStream_t st) {
    CUtensorMap mA, mB;
    if (!make_map_2d(&mA, A, p.K, p.rows, (uint64_t)p.K * 2, 64, a_rows_for(p.rows), CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&mB, B, p.K, p.N, (uint64_t)p.K * 2, 64, kLinNT, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    auto kern = linear_kernel<kLinNT, kLinStages>;
    cudaError_t e = set_smem(kern, LinC::kSmem, g_smem_linear);
    if (e != cudaSuccess) return e;
    LinArgs a;
    memset(&a, 0, sizeof(a));
    a.rows = p.rows;
    a.N = p.N;
    a.kc_per_split = p.kc_per_split;
    a.kc_total = p.kc_total;
    a.a_rows = a_rows_for(p.rows);
    a.part = part;  // fp32 partials when given, else bf16 into `out`
    a.out = out;
    a.status = status;
    a.wait_limit_ns = MLA_WAIT_LIMIT_NS;
    return launch_pdl(kern, dim3(p.col_tiles, p.splits, p.row_tiles), dim3(128), LinC::kSmem, st, 1, mA, mB, a);
}

// One warp per token: adds the S partial rows of [c || k] in split order,
// RMSNorm of the 512 latent values (fp32, eps 1e-6) times gamma, RoPE of the
// 64-wide key at the token's position; writes the bf16 cache row.  Lane l
// holds latent columns 4(l + 32j)..+3 (j < 4) and RoPE pair l.
__global__ void __launch_bounds__(256) append_hidden_finish_kernel(const float* __restrict__ part, int S, int rows,
                                                                   int n_tok, const __nv_bfloat16* __restrict__ gamma,
                                                                   const int32_t* __restrict__ pos, CacheView cache,
                                                                   RopeTable rope, int* status) {
    pdl_wait();
    pdl_trigger();
    const int row = (blockIdx.x * blockDim.x + threadIdx.x) / 32;
    const int lane = threadIdx.x % 32;
    if (row >= rows) return;
    const int b = row / n_tok, i = row % n_tok;
    const int p0 = pos[b];
    if (p0 < 0 || p0 + n_tok > cache.T_max) {
        if (lane == 0 && i == 0) atomicOr(status, MLA_STATUS_BAD_POS);
        return;
    }
    float4 c[4];
    float2 k = make_float2(0.f, 0.f);
#pragma unroll
    for (int j = 0; j < 4; ++j) c[j] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < S; ++s) {
        const float* src = part + ((size_t)s * rows + row) * kAppendRow;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float4 v = __ldg(reinterpret_cast<const float4*>(src) + lane + 32 * j);
            c[j].x += v.x; c[j].y += v.y; c[j].z += v.z; c[j].w += v.w;
        }
        const float2 v = __ldg(reinterpret_cast<const float2*>(src + kLat) + lane);
        k.x += v.x;
        k.y += v.y;
    }
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) ss += c[j].x * c[j].x + c[j].y * c[j].y + c[j].z * c[j].z + c[j].w * c[j].w;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = 1.0f / sqrtf(ss / (float)kLat + kRmsEps);
    const int t = p0 + i;
    __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(cache.data) + (size_t)b * cache.stride_b + (size_t)t * cache.stride_t;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int col = 4 * (lane + 32 * j);
        const uint2 g = *reinterpret_cast<const uint2*>(gamma + col);
        const float g0 = __uint_as_float(g.x << 16), g1 = __uint_as_float(g.x & 0xffff0000u);
        const float g2 = __uint_as_float(g.y << 16), g3 = __uint_as_float(g.y & 0xffff0000u);
        uint2 o;
        o.x = pack_bf16(c[j].x * inv * g0, c[j].y * inv * g1);
        o.y = pack_bf16(c[j].z * inv * g2, c[j].w * inv * g3);
        *reinterpret_cast<uint2*>(dst + col) = o;
    }
    float y0, y1;
    mla_rope_rotate(k.x, k.y, rope.inv_freq[lane], t, &y0, &y1);
    reinterpret_cast<__nv_bfloat162*>(dst + kLat)[lane] = __floats2bfloat162_rn(y0, y1);
}

// y = bf16(sum over the S partials in split order); eight values a thread.
__global__ void __launch_bounds__(256) sum_partials_kernel(const float* __restrict__ part, int S, size_t count,
                                                           __nv_bfloat16* __restrict__ y) {
    pdl_wait();
    pdl_trigger();
    const size_t i8 = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) * 8;
    if (i8 >= count) return;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    for (int s = 0; s < S; ++s) {
        const float4* src = reinterpret_cast<const float4*>(part + (size_t)s * count + i8);
        const float4 u = __ldg(src), v = __ldg(src + 1);
        a.x += u.x; a.y += u.y; a.z += u.z; a.w += u.w;
        b.x += v.x; b.y += v.y; b.z += v.z; b.w += v.w;
    }
    *reinterpret_cast<uint4*>(y + i8) = make_uint4(pack_bf16(a.x, a.y), pack_bf16(a.z, a.w), pack_bf16(b.x, b.y),
                                                   pack_bf16(b.z, b.w));
}

}  // namespace

// Shape rules shared by the entry points (bf16, V3 head geometry).
static bool linear_supported(const Problem& p) {
    return p.dtype == MLA_DTYPE_BF16 && p.H == kHeads && p.d_c == kLat && p.d_r == kRope && p.d_n == 128 &&
           p.d_v == 128 && sm100_supported(p, 1);
}

size_t append_hidden_workspace(int rows, int d_model) {
    const LinPlan lp = lin_plan(rows, kAppendRow, d_model);
    return (size_t)lp.splits * rows * kAppendRow * 4 + 256;
}

size_t output_projection_workspace(const Problem& p, int rows, int d_model) {
    return lin_partial_bytes(lin_plan(rows, d_model, p.H * p.d_v)) + 256;
}

cudaError_t sm100_append_hidden(const Problem& p, const void* x, const void* W_A, const void* gamma,
                                const int32_t* pos, int n_tok, int d_model, const CacheView& cache, void* ws,
                                int* status, cudaStream_t st) {
    const int rows = p.B * n_tok;
    const LinPlan lp = lin_plan(rows, kAppendRow, d_model);
    // fp32 partials even for one split: the epilogue normalises the whole
    // unrounded row
    float* part = static_cast<float*>(ws);
    cudaError_t e = lin_launch(lp, x, W_A, part, nullptr, status, st);
    if (e != cudaSuccess) return e;
    const int threads = 256;
    const int blocks = (rows * 32 + threads - 1) / threads;
    return launch_pdl(append_hidden_finish_kernel, dim3(blocks), dim3(threads), 0, st, 1, (const float*)part,
                      lp.splits, rows, n_tok, (const __nv_bfloat16*)gamma, pos, cache, p.rope, status);
}

cudaError_t sm100_output_projection(const Problem& p, const void* attn_out, const void* W_O, int rows, int d_model,
                                    void* y, void* ws, int* status, cudaStream_t st) {
    const LinPlan lp = lin_plan(rows, d_model, p.H * p.d_v);
    if (lp.splits == 1) return lin_launch(lp, attn_out, W_O, nullptr, (__nv_bfloat16*)y, status, st);
    float* part = static_cast<float*>(ws);
    cudaError_t e = lin_launch(lp, attn_out, W_O, part, nullptr, status, st);
    if (e != cudaSuccess) return e;
    const size_t count = (size_t)rows * d_model;
    const int threads = 256;
    const unsigned blocks = (unsigned)((count / 8 + threads - 1) / threads);
    return launch_pdl(sum_partials_kernel, dim3(blocks), dim3(threads), 0, st, 1, (const float*)part, lp.splits, count,
                      (__nv_bfloat16*)y);
}

bool sm100_linear_supported(const Problem& p) { return linear_supported(p); }

}  // namespace mla
