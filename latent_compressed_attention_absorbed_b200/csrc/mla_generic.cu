// Generic CUDA-core kernels for absorbed MLA decode: any head geometry, fp32
// or bf16 storage, fp32 arithmetic.  They serve shapes the sm_100a
// tensor-core kernels do not cover (e.g. the 4-head fp32 case) and act as an
// independent second GPU implementation in tests.  Throughput is not their
// purpose.
//
// Method references (see include/mla.h): cache row = [c_KV || RoPE(k_R)]
// (092 page, section 二 "MLA：缓存压缩后的历史"); q_lat = W_UK^T q_nope and the
// RoPE score added separately (092 page, "缓存压缩也可以做一个代数检查";
// m.lsln.cn sections 2.2-2.3); aggregate in latent space then apply W_UV
// (ailearn.mscapital.top MLA panel).
#include <cuda_bf16.h>
#include <math.h>

#include "mla_internal.h"
#include "mla_rope.cuh"

namespace mla {
namespace {

__device__ __forceinline__ float ld(const float* p, size_t i) { return p[i]; }
__device__ __forceinline__ float ld(const __nv_bfloat16* p, size_t i) { return __bfloat162float(p[i]); }
__device__ __forceinline__ void st(float* p, size_t i, float v) { p[i] = v; }
__device__ __forceinline__ void st(__nv_bfloat16* p, size_t i, float v) { p[i] = __float2bfloat16_rn(v); }

template <typename T>
__global__ void append_kernel(Problem p, const T* __restrict__ c_kv, const T* __restrict__ k_rope,
                              const int32_t* __restrict__ pos, int n_tok, CacheView cache, int* status) {
    const int b = blockIdx.x / n_tok, i = blockIdx.x % n_tok;
    const int p0 = pos[b];
    const int t = p0 + i;
    if (p0 < 0 || p0 + n_tok > cache.T_max) {
        if (threadIdx.x == 0 && i == 0) atomicOr(status, MLA_STATUS_BAD_POS);
        return;
    }
    T* row = static_cast<T*>(cache.data) + (size_t)b * cache.stride_b + (size_t)t * cache.stride_t;
    const T* c = c_kv + ((size_t)b * n_tok + i) * p.d_c;
    const T* k = k_rope + ((size_t)b * n_tok + i) * p.d_r;
    for (int e = threadIdx.x; e < p.d_c; e += blockDim.x) row[e] = c[e];
    for (int kk = threadIdx.x; kk < p.d_r / 2; kk += blockDim.x) {
        float y0, y1;
        mla_rope_rotate(ld(k, 2 * kk), ld(k, 2 * kk + 1), p.rope.inv_freq[kk], t, &y0, &y1);
        st(row, p.d_c + 2 * kk, y0);
        st(row, p.d_c + 2 * kk + 1, y1);
    }
}

// q_hat[u][h] = [W_UK[h]^T q_nope[u][h] || RoPE(q_rope[u][h], m)]; one block per (u, h).
template <typename T>
__global__ void absorb_kernel(Problem p, const T* __restrict__ q_nope, const T* __restrict__ q_rope,
                              const T* __restrict__ W_UK, const int32_t* __restrict__ seqlens,
                              T* __restrict__ q_hat) {
    extern __shared__ float sq[];
    const int u = blockIdx.x / p.H, h = blockIdx.x % p.H;
    const int b = u / p.q_len, i = u % p.q_len;
    const T* qn = q_nope + ((size_t)u * p.H + h) * p.d_n;
    for (int d = threadIdx.x; d < p.d_n; d += blockDim.x) sq[d] = ld(qn, d);
    __syncthreads();
    T* out = q_hat + ((size_t)u * p.H + h) * (p.d_c + p.d_r);
    const T* W = W_UK + (size_t)h * p.d_n * p.d_c;
    for (int c = threadIdx.x; c < p.d_c; c += blockDim.x) {
        float acc = 0.f;
        for (int d = 0; d < p.d_n; ++d) acc = fmaf(sq[d], ld(W, (size_t)d * p.d_c + c), acc);
        st(out, c, acc);
    }
    const int m = seqlens[b] - p.q_len + i;
    const T* qr = q_rope + ((size_t)u * p.H + h) * p.d_r;
    for (int kk = threadIdx.x; kk < p.d_r / 2; kk += blockDim.x) {
        float y0, y1;
        mla_rope_rotate(ld(qr, 2 * kk), ld(qr, 2 * kk + 1), p.rope.inv_freq[kk], m, &y0, &y1);
        st(out, p.d_c + 2 * kk, y0);
        st(out, p.d_c + 2 * kk + 1, y1);
    }
}

constexpr int kAttWarps = 8;
constexpr int kMaxPerLane = 32;  // d_c <= 1024

// One block per (u, h).  Each warp runs an online softmax over keys
// j = warp, warp + 8, ...; the eight partial states are merged at the end.
template <typename T>
__global__ void __launch_bounds__(kAttWarps * 32) attend_kernel(Problem p, const T* __restrict__ q_hat,
                                                                CacheView cache, const int32_t* __restrict__ seqlens,
                                                                T* __restrict__ o_lat, int* status) {
    extern __shared__ float smem[];
    const int row = p.d_c + p.d_r;
    float* sq = smem;                         // [row]
    float* sm = sq + row;                     // [warps] running max
    float* sl = sm + kAttWarps;               // [warps] running sum
    float* so = sl + kAttWarps;               // [warps][d_c]
    const int u = blockIdx.x / p.H, h = blockIdx.x % p.H;
    const int b = u / p.q_len, i = u % p.q_len;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int T_b = seqlens[b];
    T* out = o_lat + ((size_t)u * p.H + h) * p.d_c;
    if (T_b < p.q_len || T_b > cache.T_max) {
        if (threadIdx.x == 0) atomicOr(status, MLA_STATUS_BAD_SEQLEN);
        for (int c = threadIdx.x; c < p.d_c; c += blockDim.x) st(out, c, 0.f);
        return;
    }
    const int n_keys = T_b - p.q_len + 1 + i;
    const T* q = q_hat + ((size_t)u * p.H + h) * row;
    for (int e = threadIdx.x; e < row; e += blockDim.x) sq[e] = ld(q, e);
    __syncthreads();

    const T* base = static_cast<const T*>(cache.data) + (size_t)b * cache.stride_b;
    float m_run = -INFINITY, l_run = 0.f;
    float acc[kMaxPerLane];
#pragma unroll
    for (int r = 0; r < kMaxPerLane; ++r) acc[r] = 0.f;
    for (int j = warp; j < n_keys; j += kAttWarps) {
        const T* kr = base + (size_t)j * cache.stride_t;
        float s = 0.f;
        for (int e = lane; e < row; e += 32) s = fmaf(sq[e], ld(kr, e), s);
#pragma unroll
        for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        s *= p.scale;
        const float m_new = fmaxf(m_run, s);
        const float corr = __expf(m_run - m_new);
        const float pj = __expf(s - m_new);
        l_run = l_run * corr + pj;
#pragma unroll
        for (int r = 0; r < kMaxPerLane; ++r) {
            const int c = lane + 32 * r;
            if (c < p.d_c) acc[r] = acc[r] * corr + pj * ld(kr, c);
        }
        m_run = m_new;
    }
    if (lane == 0) {
        sm[warp] = m_run;
        sl[warp] = l_run;
    }
#pragma unroll
    for (int r = 0; r < kMaxPerLane; ++r) {
        const int c = lane + 32 * r;
        if (c < p.d_c) so[warp * p.d_c + c] = acc[r];
    }
    __syncthreads();
    float M = -INFINITY;
    for (int w = 0; w < kAttWarps; ++w) M = fmaxf(M, sm[w]);
    float L = 0.f;
    for (int w = 0; w < kAttWarps; ++w) L += (sm[w] == -INFINITY) ? 0.f : sl[w] * __expf(sm[w] - M);
    for (int c = threadIdx.x; c < p.d_c; c += blockDim.x) {
        float o = 0.f;
        for (int w = 0; w < kAttWarps; ++w)
            if (sm[w] != -INFINITY) o += so[w * p.d_c + c] * __expf(sm[w] - M);
        st(out, c, o / L);
    }
}

// out[r][h][d] = sum_c W_UV[h][d][c] o_lat[r][h][c]; one block per (r, h), one warp per output d.
template <typename T>
__global__ void project_kernel(Problem p, const T* __restrict__ o_lat, const T* __restrict__ W_UV,
                               T* __restrict__ out) {
    extern __shared__ float so[];
    const int r = blockIdx.x / p.H, h = blockIdx.x % p.H;
    const T* o = o_lat + ((size_t)r * p.H + h) * p.d_c;
    for (int c = threadIdx.x; c < p.d_c; c += blockDim.x) so[c] = ld(o, c);
    __syncthreads();
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, nw = blockDim.x / 32;
    const T* W = W_UV + (size_t)h * p.d_v * p.d_c;
    for (int d = warp; d < p.d_v; d += nw) {
        float acc = 0.f;
        for (int c = lane; c < p.d_c; c += 32) acc = fmaf(ld(W, (size_t)d * p.d_c + c), so[c], acc);
#pragma unroll
        for (int k = 16; k; k >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, k);
        if (lane == 0) st(out, ((size_t)r * p.H + h) * p.d_v + d, acc);
    }
}

}  // namespace

#define MLA_DISPATCH(p, F, ...)                                                          \
    ((p).dtype == MLA_DTYPE_F32 ? F<float>(__VA_ARGS__) : F<__nv_bfloat16>(__VA_ARGS__))

template <typename T>
static cudaError_t append_t(const Problem& p, const void* c_kv, const void* k_rope, const int32_t* pos, int n_tok,
                            const CacheView& cache, int* status, cudaStream_t st) {
    append_kernel<T><<<p.B * n_tok, 128, 0, st>>>(p, (const T*)c_kv, (const T*)k_rope, pos, n_tok, cache, status);
    return cudaGetLastError();
}
cudaError_t generic_append(const Problem& p, const void* c_kv, const void* k_rope, const int32_t* pos, int n_tok,
                           const CacheView& cache, int* status, cudaStream_t st) {
    return MLA_DISPATCH(p, append_t, p, c_kv, k_rope, pos, n_tok, cache, status, st);
}

template <typename T>
static cudaError_t absorb_t(const Problem& p, const void* q_nope, const void* q_rope, const void* W_UK,
                            const int32_t* seqlens, void* q_hat, cudaStream_t st) {
    absorb_kernel<T><<<p.B * p.q_len * p.H, 256, p.d_n * sizeof(float), st>>>(
        p, (const T*)q_nope, (const T*)q_rope, (const T*)W_UK, seqlens, (T*)q_hat);
    return cudaGetLastError();
}
cudaError_t generic_absorb(const Problem& p, const void* q_nope, const void* q_rope, const void* W_UK,
                           const int32_t* seqlens, void* q_hat, cudaStream_t st) {
    return MLA_DISPATCH(p, absorb_t, p, q_nope, q_rope, W_UK, seqlens, q_hat, st);
}

template <typename T>
static cudaError_t attend_t(const Problem& p, const void* q_hat, const CacheView& cache, const int32_t* seqlens,
                            void* o_lat, int* status, cudaStream_t st) {
    const size_t smem = sizeof(float) * ((p.d_c + p.d_r) + 2 * kAttWarps + (size_t)kAttWarps * p.d_c);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(attend_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    attend_kernel<T><<<p.B * p.q_len * p.H, kAttWarps * 32, smem, st>>>(p, (const T*)q_hat, cache, seqlens, (T*)o_lat,
                                                                         status);
    return cudaGetLastError();
}
cudaError_t generic_attend(const Problem& p, const void* q_hat, const CacheView& cache, const int32_t* seqlens,
                           void* o_lat, int* status, cudaStream_t st) {
    if (p.d_c > 32 * kMaxPerLane) return cudaErrorInvalidValue;
    return MLA_DISPATCH(p, attend_t, p, q_hat, cache, seqlens, o_lat, status, st);
}

template <typename T>
static cudaError_t project_t(const Problem& p, const void* o_lat, const void* W_UV, int rows, void* out,
                             cudaStream_t st) {
    project_kernel<T><<<rows * p.H, 256, p.d_c * sizeof(float), st>>>(p, (const T*)o_lat, (const T*)W_UV, (T*)out);
    return cudaGetLastError();
}
cudaError_t generic_project(const Problem& p, const void* o_lat, const void* W_UV, int rows, void* out,
                            cudaStream_t st) {
    return MLA_DISPATCH(p, project_t, p, o_lat, W_UV, rows, out, st);
}

size_t generic_workspace_bytes(const Problem& p) {
    const size_t es = p.dtype == MLA_DTYPE_F32 ? 4 : 2;
    const size_t U = (size_t)p.B * p.q_len * p.H;
    Carve c(nullptr);
    c.take(U * (p.d_c + p.d_r) * es);  // q_hat
    c.take(U * p.d_c * es);            // o_lat
    return c.off;
}

}  // namespace mla
