// The two per-head projections of absorbed MLA for small batches (at most
// eight query tokens), where they are matrix-vector products bound by the
// weight reads (16.8 MB each):
//
//   absorb  (a2): q_lat[u][h][:] = W_UK[h]^T q_nope[u][h][:]   (128 -> 512)
//                 plus the RoPE of q_R at the query position
//   project (a5): out[u][h][:]   = W_UV[h] o_lat[u][h][:]      (512 -> 128)
//
// (092 page, section 二 "缓存压缩也可以做一个代数检查": fold U^T into the query
// once; ailearn.mscapital.top MLA panel: W_UV after the latent aggregation.)
//
// Each CTA stages its slice of the weights in shared memory with TMA (one
// 64 KB box for absorb, eight 16 KB boxes for project, all completing on one
// mbarrier) before waiting for the previous kernel (weights are never
// written by it), so the weight stream overlaps the previous kernel's tail.
// The project kernel also merges the split-KV partials of the attention
// step itself (so the decode needs no separate combine launch for these
// batches).
#pragma once

#include <cuda_bf16.h>
#include <math_constants.h>

#include "mla_rope.cuh"
#include "sm100_attend.cuh"
#include "sm100_ptx.cuh"

namespace mla {
namespace sm100 {

constexpr int kGemvMaxRows = 8;
constexpr int kGemvWBytes = 64 * 1024;  // weight slice of one CTA
// + the mbarrier (16 bytes) and slack to align the TMA destination to 128 bytes
template <int R> constexpr int absorb_gemv_smem() { return kGemvWBytes + R * 128 * 4 + 16 + 128; }
constexpr int kMergeStateFloats = kLat + 4;  // acc[512], m, wsum (padded)
constexpr int kProjWarps = 16;                 // project CTA: 512 threads, all 128 output rows of a head
// W_UV[h] in shared memory: eight SW128 boxes of 64 latent columns x 128 rows
// (row v's 16-byte chunk c of box k at k*16 KB + v*128 + ((c ^ (v % 8)) * 16),
// so the eight rows a quarter-warp reads at once hit distinct banks)
constexpr int kProjWBytes = 128 * kLat * 2;    // 128 KB
template <int R> constexpr int project_gemv_smem() {
    return kProjWBytes + R * kLat * 4 + kProjWarps * kMergeStateFloats * 4 + 4 * R * 128 * 4 + 16 + 1024;
}


__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t v) {
    return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
}

struct AbsorbGemvArgs {
    const __nv_bfloat16* q_nope;  // [rows][128][128]
    const __nv_bfloat16* q_rope;  // [rows][128][64]
    const __nv_bfloat16* W_UK;    // [128][128][512]
    const int32_t* seqlens;       // [B]
    int rows, q_len;
    __nv_bfloat16* q_hat;         // [rows][128][576]
    RopeTable rope;
    int* status;
    // split plan of the attention step, written by CTA (128, 0)
    Plan* plan;
    int plan_B, plan_T_max, plan_clusters, plan_ovh, plan_min_units;
    __nv_bfloat16* plan_olat;
};

// grid (129, 2), 128 threads: CTA (h, y) produces latent columns
// 256y..256y+255 of head h for every row and RoPE pairs 16y..16y+15; CTA
// (128, 0) writes the attention plan.  Thread t owns columns 2t, 2t+1.
// mapW: W_UK as [128 heads][128 d][512 c] bf16, box 256 c x 128 d, no swizzle
// (the box lands as w_s[d][256]).
template <int R>
__global__ void __launch_bounds__(128) absorb_gemv_kernel(const __grid_constant__ CUtensorMap mapW, AbsorbGemvArgs a) {
    extern __shared__ __align__(16) uint8_t gemv_smem_raw[];
    uint8_t* gemv_smem = gemv_smem_raw + ((128u - (smem_u32(gemv_smem_raw) & 127u)) & 127u);
    auto w_s = reinterpret_cast<__nv_bfloat16(*)[256]>(gemv_smem);                 // W_UK[h][d][256y ..]
    auto q_s = reinterpret_cast<float(*)[128]>(gemv_smem + kGemvWBytes);          // q_nope rows, fp32
    const uint32_t wbar = smem_u32(gemv_smem + kGemvWBytes + R * 128 * 4);
    const int h = blockIdx.x, y = blockIdx.y, t = threadIdx.x;
    MLA_KT(kKtAbsorb, 0);
    if (h == kHeads) {
        pdl_wait();
        if (y == 0 && t < 32 && a.plan)
            mla_plan_warp(a.seqlens, a.plan_B, a.q_len, a.plan_T_max, a.plan_clusters, a.plan_ovh,
                          a.plan_min_units, a.plan, a.status, a.plan_olat, t);
        if (t == 0) pdl_trigger();
        MLA_KT(kKtAbsorb, 2);
        return;
    }
    // weights first (they do not depend on the previous kernel): one 64 KB box
    if (t == 0) {
        mbar_init(wbar, 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(wbar, kGemvWBytes);
        tma_load_3d(smem_u32(&w_s[0][0]), &mapW, wbar, 256 * y, 0, h);
    }
    pdl_wait();
    if (t == 0) pdl_trigger();
    MLA_KT(kKtAbsorb, 1);
    for (int i = t; i < R * 128; i += 128) {
        const int u = i / 128, d = i % 128;
        q_s[u][d] = u < a.rows ? __bfloat162float(a.q_nope[((size_t)u * kHeads + h) * 128 + d]) : 0.f;
    }
    // RoPE of q_R at the query position m = T_b - q_len + i (pairs 16y..16y+15)
    if (t < R * 16) {
        const int u = t / 16, k = 16 * y + t % 16;
        if (u < a.rows) {
            const int b = u / a.q_len, i = u % a.q_len;
            const int m = a.seqlens[b] - a.q_len + i;
            const __nv_bfloat162 x =
                reinterpret_cast<const __nv_bfloat162*>(a.q_rope + ((size_t)u * kHeads + h) * kRope)[k];
            float y0, y1;
            mla_rope_rotate(__low2float(x), __high2float(x), a.rope.inv_freq[k], m, &y0, &y1);
            reinterpret_cast<__nv_bfloat162*>(a.q_hat + ((size_t)u * kHeads + h) * kRow + kLat)[k] =
                __floats2bfloat162_rn(y0, y1);
        }
    }
    __syncthreads();  // q_s, and the barrier's initialisation, are visible to every thread
    if (!mbar_wait(wbar, 0, MLA_WAIT_LIMIT_NS)) {
        atomicOr(a.status, MLA_STATUS_TIMEOUT);
        mbar_wait(wbar, 0, MLA_WAIT_LIMIT_NS);  // the copy must not land after the CTA has exited
        return;
    }
    float acc[R][2];
#pragma unroll
    for (int u = 0; u < R; ++u) acc[u][0] = acc[u][1] = 0.f;
    const uint32_t* wrow = reinterpret_cast<const uint32_t*>(&w_s[0][0]) + t;
#pragma unroll 8
    for (int d = 0; d < 128; ++d) {
        const float2 w = bf16x2_to_f2(wrow[d * 128]);
#pragma unroll
        for (int u = 0; u < R; ++u) {
            const float q = q_s[u][d];
            acc[u][0] = fmaf(w.x, q, acc[u][0]);
            acc[u][1] = fmaf(w.y, q, acc[u][1]);
        }
    }
#pragma unroll
    for (int u = 0; u < R; ++u)
        if (u < a.rows)
            reinterpret_cast<__nv_bfloat162*>(a.q_hat + ((size_t)u * kHeads + h) * kRow + 256 * y)[t] =
                __floats2bfloat162_rn(acc[u][0], acc[u][1]);
    MLA_KT(kKtAbsorb, 2);
}

struct ProjectGemvArgs {
    const Plan* plan;             // split plan (decode path)
    const __nv_bfloat16* o_lat;   // [rows][128][512]: unsplit units (and zeroed invalid ones)
    const float* part_o;          // [slots][128][512]
    const float* part_lse;        // [slots][128]
    const __nv_bfloat16* W_UV;    // [128][128][512]
    int rows;
    __nv_bfloat16* out;           // [rows][128][128]
    int* status;
};

// grid (128), 512 threads: CTA h produces all 128 output columns of head h.
// With R rows and G = 16 / R warps per row, warp w serves row u = w % R as
// member g = w / R of its group:
//   1. o_lat of row u in fp32: read directly (unit not split), or merged from
//      the split partials, each warp of the group taking every G-th piece and
//      the group's states combined through shared memory;
//   2. thread (v, q) forms the dot products of output row v with every row
//      over latent columns 128q..128q+127; the four partial sums are added
//      through shared memory.
// mapW: W_UV as [128 heads][128 v][512 c] bf16, box 64 c x 128 v, SW128.
template <int R>
__global__ void __launch_bounds__(512) project_gemv_kernel(const __grid_constant__ CUtensorMap mapW, ProjectGemvArgs a) {
    constexpr int G = kProjWarps / R;
    extern __shared__ __align__(16) uint8_t gemv_smem_raw[];
    uint8_t* gemv_smem = gemv_smem_raw + ((1024u - (smem_u32(gemv_smem_raw) & 1023u)) & 1023u);
    uint8_t* w_s = gemv_smem;                                                          // W_UV[h], eight SW128 boxes
    auto o_s = reinterpret_cast<float(*)[kLat]>(gemv_smem + kProjWBytes);              // o_lat rows, fp32
    auto st_s = reinterpret_cast<float(*)[kMergeStateFloats]>(gemv_smem + kProjWBytes + R * kLat * 4);
    auto sum_s = reinterpret_cast<float(*)[R][128]>(gemv_smem + kProjWBytes + R * kLat * 4 +
                                                     kProjWarps * kMergeStateFloats * 4);  // [4 column quarters][R][v]
    const int h = blockIdx.x, t = threadIdx.x;
    const int warp = t / 32, lane = t % 32;
    const int u = warp % R, g = warp / R;
    MLA_KT(kKtProject, 0);
    const uint32_t wbar = smem_u32(gemv_smem + kProjWBytes + R * kLat * 4 + kProjWarps * kMergeStateFloats * 4 +
                                   4 * R * 128 * 4);
    if (t == 0) {
        mbar_init(wbar, 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(wbar, kProjWBytes);
#pragma unroll 1
        for (int k = 0; k < 8; ++k) tma_load_3d(smem_u32(w_s) + k * 16384, &mapW, wbar, 64 * k, 0, h);
    }
    pdl_wait();
    if (t == 0) pdl_trigger();
    MLA_KT(kKtProject, 1);
    // ---- 1. o_lat of row u
    bool split = false;
    UnitPieces up;
    int b = 0, qi = 0, q_len = 1;
    if (u < a.rows && a.plan) {
        q_len = a.plan->q_len;
        b = u / q_len;
        qi = u % q_len;
        up.init(a.plan, b);
        split = up.split;
    }
    if (split) {
        MergeState ms;
        ms.clear();
        merge_pieces_warp(up, b, qi, q_len, h, a.part_o, a.part_lse, lane, g, G, ms);
#pragma unroll
        for (int j = 0; j < 4; ++j) reinterpret_cast<float4*>(&st_s[warp][0])[lane + 32 * j] = ms.acc[j];
        if (lane == 0) {
            st_s[warp][kLat] = ms.m;
            st_s[warp][kLat + 1] = ms.wsum;
        }
    } else if (g == 0) {
        const uint2* src = reinterpret_cast<const uint2*>(a.o_lat + ((size_t)u * kHeads + h) * kLat) + lane;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint2 v = u < a.rows ? src[32 * j] : make_uint2(0, 0);
            const float2 lo = bf16x2_to_f2(v.x), hi = bf16x2_to_f2(v.y);
            reinterpret_cast<float4*>(&o_s[u][0])[lane + 32 * j] = make_float4(lo.x, lo.y, hi.x, hi.y);
        }
    }
    __syncthreads();
    if (split && g == 0) {
        MergeState ms;
        ms.clear();
        for (int k = 0; k < G; ++k) {
            const int wk = u + R * k;
            float4 a2[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) a2[j] = reinterpret_cast<const float4*>(&st_s[wk][0])[lane + 32 * j];
            ms.fold(st_s[wk][kLat], st_s[wk][kLat + 1], a2);
        }
        ms.normalise();
        // the merged value is what the unsplit path holds: bf16 o_lat
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 lo = bf16x2_to_f2(pack_bf16(ms.acc[j].x, ms.acc[j].y));
            const float2 hi = bf16x2_to_f2(pack_bf16(ms.acc[j].z, ms.acc[j].w));
            reinterpret_cast<float4*>(&o_s[u][0])[lane + 32 * j] = make_float4(lo.x, lo.y, hi.x, hi.y);
        }
    }
    __syncthreads();  // o_s, and the barrier's initialisation, are visible to every thread
    const bool w_ok = mbar_wait(wbar, 0, MLA_WAIT_LIMIT_NS);
    // ---- 2. out[u][h][v] = sum_c W_UV[h][v][c] o[u][c]: thread (v, quarter q) takes
    // output row v = t % 128 and latent columns 128q..128q+127 (boxes 2q, 2q+1)
    // for every row u; the four quarters are added through shared memory.
    {
        const int v = t % 128, q = t / 128;
        float acc[R];
#pragma unroll
        for (int uu = 0; uu < R; ++uu) acc[uu] = 0.f;
        const uint8_t* wrow = w_s + 2 * q * 16384 + v * 128;
#pragma unroll 2
        for (int c8 = 0; c8 < 16 && w_ok; ++c8) {
            const uint4 w8 =
                *reinterpret_cast<const uint4*>(wrow + (c8 >> 3) * 16384 + (((c8 & 7) ^ (v & 7)) << 4));
            const float2 w01 = bf16x2_to_f2(w8.x), w23 = bf16x2_to_f2(w8.y);
            const float2 w45 = bf16x2_to_f2(w8.z), w67 = bf16x2_to_f2(w8.w);
#pragma unroll
            for (int uu = 0; uu < R; ++uu) {
                const float4 o0 = *reinterpret_cast<const float4*>(&o_s[uu][128 * q + 8 * c8]);
                const float4 o1 = *reinterpret_cast<const float4*>(&o_s[uu][128 * q + 8 * c8 + 4]);
                float x = acc[uu];
                x = fmaf(w01.x, o0.x, x); x = fmaf(w01.y, o0.y, x);
                x = fmaf(w23.x, o0.z, x); x = fmaf(w23.y, o0.w, x);
                x = fmaf(w45.x, o1.x, x); x = fmaf(w45.y, o1.y, x);
                x = fmaf(w67.x, o1.z, x); x = fmaf(w67.y, o1.w, x);
                acc[uu] = x;
            }
        }
#pragma unroll
        for (int uu = 0; uu < R; ++uu) sum_s[q][uu][v] = acc[uu];
    }
    __syncthreads();
    for (int i = t; i < R * 128; i += 512) {
        const int uu = i / 128, v = i % 128;
        if (uu < a.rows)
            a.out[((size_t)uu * kHeads + h) * 128 + v] =
                __float2bfloat16_rn(sum_s[0][uu][v] + sum_s[1][uu][v] + sum_s[2][uu][v] + sum_s[3][uu][v]);
    }
    if (!w_ok && t == 0) {
        atomicOr(a.status, MLA_STATUS_TIMEOUT);
        mbar_wait(wbar, 0, MLA_WAIT_LIMIT_NS);  // the copies must not land after the CTA has exited
    }
    MLA_KT(kKtProject, 2);
}

}  // namespace sm100
}  // namespace mla
