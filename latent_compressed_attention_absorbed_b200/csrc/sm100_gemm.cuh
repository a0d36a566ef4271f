// Per-head batched GEMM on tcgen05 for the two projections of absorbed MLA.
//
//   absorb  (a2): q_lat[u][h][:] = W_UK[h]^T q_nope[u][h][:]   M=rows, N=512, K=128
//           W_UK[h] is [d_n=K][d_c=N] with N contiguous  -> B operand MN-major
//   project (a5): out[u][h][:]   = W_UV[h] o_lat[u][h][:]      M=rows, N=128, K=512
//           W_UV[h] is [d_v=N][d_c=K] with K contiguous  -> B operand K-major
//
// (092 page, section 二 "缓存压缩也可以做一个代数检查": fold U^T into the query
// once; ailearn.mscapital.top MLA panel: W_UV after the latent aggregation.)
//
// One CTA computes a 128-row x NT-column tile of one head.  Warp 0 issues TMA
// loads into a STAGES-deep ring of K-chunks (64 wide), warp 1 allocates TMEM
// and issues tcgen05.mma (M=128, N=NT, K=16 each), then all four warps drain
// the fp32 accumulator from TMEM and store bf16.  The absorb variant also
// rotates q_R (RoPE at the query position) in its column-0 CTAs.
#pragma once

#include <cuda_bf16.h>

#include "mla_rope.cuh"
#include "sm100_attend.cuh"
#include "sm100_ptx.cuh"

namespace mla {
namespace sm100 {

struct GemmArgs {
    int rows;         // M extent (query tokens)
    int H;            // heads
    int ld_out;       // output row stride (elements) per (u, h)
    int out_col0;     // first output column of this GEMM inside the row
    __nv_bfloat16* out;
    // RoPE part of the absorb step (ignored when !ROPE)
    const __nv_bfloat16* q_rope;  // [rows][H][64]
    const int32_t* seqlens;       // [B]
    int q_len;
    RopeTable rope;
    int a_rows;       // rows of each A box (multiple of 16, <= 128)
    int out_v8;       // out is 32-byte aligned: 32-byte stores in the epilogue
    int* status;
    // split plan of the attention step, written by warp 2 of CTA (0,0,0) when non-null
    Plan* plan;
    int plan_B, plan_T_max, plan_clusters, plan_ovh, plan_min_units;
    __nv_bfloat16* plan_olat;
};

template <int KCH, int NT, bool B_MN, int STAGES, bool ROPE>
struct GemmCfg {
    static constexpr int kABytes = 128 * 128;           // 128 rows x 64 bf16
    static constexpr int kBBytes = NT * 128;            // NT x 64 bf16
    static constexpr int kStage = kABytes + kBBytes;
    static constexpr int kSmem = STAGES * kStage + 1024 /*barriers*/ + 1024 /*align*/;
    static constexpr int kTmemCols = NT < 32 ? 32 : NT;
    static constexpr uint32_t kIdesc = idesc_bf16_f32(128, NT, false, B_MN);
};

template <int KCH, int NT, bool B_MN, int STAGES, bool ROPE>
__global__ void __launch_bounds__(128, 1)
    head_gemm_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                     GemmArgs args) {
    using C = GemmCfg<KCH, NT, B_MN, STAGES, ROPE>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* base_ptr = smem_raw + (base - raw);
    const uint32_t bars = base + STAGES * C::kStage;
    auto full_bar = [&](int s) { return bars + 8u * s; };
    auto empty_bar = [&](int s) { return bars + 8u * (STAGES + s); };
    const uint32_t done_bar = bars + 8u * (2 * STAGES);
    const uint32_t tmem_slot = bars + 8u * (2 * STAGES + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(base_ptr + STAGES * C::kStage + 8 * (2 * STAGES + 2));

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int h = blockIdx.x;
    const int n0 = blockIdx.y * NT;
    MLA_KT(ROPE ? kKtAbsorb : kKtProject, 0);
    const int m0 = blockIdx.z * 128;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        mbar_init(done_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&mapA);
        prefetch_tensormap(&mapB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(base_ptr + (tmem_slot - base));

    if (warp == 0 && lane == 0) {
        // ---------------- producer
        // The weight tiles (B) of the first stages are requested before the
        // grid dependency wait: weights are never written by the kernel
        // that precedes this one.  The activations (A) only after it.
        constexpr int kPre = KCH < STAGES ? KCH : STAGES;
        auto load_B = [&](int kc, int s) {
            const uint32_t b_dst = base + s * C::kStage + C::kABytes;
            if (B_MN) {
#pragma unroll
                for (int j = 0; j < NT / 64; ++j)
                    tma_load_3d(b_dst + j * 8192, &mapB, full_bar(s), n0 + 64 * j, kc * 64, h);
            } else {
                tma_load_3d(b_dst, &mapB, full_bar(s), kc * 64, n0, h);
            }
        };
        for (int kc = 0; kc < kPre; ++kc) {
            mbar_arrive_expect_tx(full_bar(kc), args.a_rows * 128 + C::kBBytes);
            load_B(kc, kc);
        }
        pdl_wait();
        pdl_trigger();
        for (int kc = 0; kc < KCH; ++kc) {
            const int s = kc % STAGES;
            if (kc >= kPre) {
                if (!mbar_wait(empty_bar(s), ((kc / STAGES) - 1) & 1)) {
                    *abort_flag = 1;
                    break;
                }
                mbar_arrive_expect_tx(full_bar(s), args.a_rows * 128 + C::kBBytes);
                load_B(kc, s);
            }
            tma_load_3d(base + s * C::kStage, &mapA, full_bar(s), kc * 64, h, m0);
        }
    } else if (warp == 1 && lane == 0) {
        // ---------------- MMA issuer
        for (int kc = 0; kc < KCH; ++kc) {
            const int s = kc % STAGES;
            if (*abort_flag || !mbar_wait(full_bar(s), (kc / STAGES) & 1)) {
                *abort_flag = 1;
                break;
            }
            tc_fence_after();
            const uint32_t a_addr = base + s * C::kStage;
            const uint32_t b_addr = a_addr + C::kABytes;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint64_t ad = smem_desc(a_addr + 32 * k, 16, 1024, kSw128);
                const uint64_t bd = B_MN ? smem_desc(b_addr + 2048 * k, 8192, 1024, kSw128)
                                         : smem_desc(b_addr + 32 * k, 16, 1024, kSw128);
                mma_f16_ss(tmem, ad, bd, C::kIdesc, (kc | k) ? 1u : 0u);
            }
            mma_commit(empty_bar(s));
        }
        mma_commit(done_bar);
    }
    // Nothing is written before the kernels this one depends on have completed.
    pdl_wait();
    MLA_KT(ROPE ? kKtAbsorb : kKtProject, 1);
    if (warp == 2 && args.plan && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0)
        mla_plan_warp(args.seqlens, args.plan_B, args.q_len, args.plan_T_max, args.plan_clusters, args.plan_ovh,
                      args.plan_min_units, args.plan, args.status, args.plan_olat, lane);
    __syncwarp();
    if (ROPE && warp >= 2) {
        // q_hat[u][h][512 + 2k..] = RoPE(q_rope[u][h], m_u) for the rows of this
        // tile, pairs 16y..16y+15 in the CTA with N-tile y, m_u = seqlens[b] -
        // q_len + i; four pairs (16 bytes) per item, four items' loads in flight
        // per thread, while the MMAs run.
        const int tid2 = threadIdx.x - 64;
        const int items = min(128, args.rows - m0) * 4;
        for (int it0 = tid2; it0 < items; it0 += 64 * 4) {
            uint4 x[4];
            int pos[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int it = it0 + 64 * j;
                if (it < items) {
                    const int u = m0 + it / 4, k0 = 16 * blockIdx.y + 4 * (it % 4);
                    x[j] = __ldg(reinterpret_cast<const uint4*>(args.q_rope + ((size_t)u * args.H + h) * 64 + 2 * k0));
                    const int b = u / args.q_len, i = u % args.q_len;
                    pos[j] = args.seqlens[b] - args.q_len + i;
                }
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int it = it0 + 64 * j;
                if (it < items) {
                    const int u = m0 + it / 4, k0 = 16 * blockIdx.y + 4 * (it % 4);
                    const uint32_t in[4] = {x[j].x, x[j].y, x[j].z, x[j].w};
                    uint32_t o[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        float y0, y1;
                        mla_rope_rotate(__uint_as_float(in[q] << 16), __uint_as_float(in[q] & 0xffff0000u),
                                        args.rope.inv_freq[k0 + q], pos[j], &y0, &y1);
                        o[q] = pack_bf16(y0, y1);
                    }
                    *reinterpret_cast<uint4*>(args.out + ((size_t)u * args.H + h) * args.ld_out + 512 + 2 * k0) =
                        make_uint4(o[0], o[1], o[2], o[3]);
                }
            }
        }
    }

    // ---------------- epilogue: all four warps, TMEM lane quarter = warp
    // warp-uniform: the TMEM loads below are whole-warp (.aligned) instructions
    const bool ok = __all_sync(0xffffffffu, mbar_wait(done_bar, 0) && !*abort_flag);
    tc_fence_after();
    const int row = m0 + warp * 32 + lane;
    if (ok) {
#pragma unroll 1
        for (int c0 = 0; c0 < NT; c0 += 32) {
            uint32_t r[32];
            tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + c0, r);
            tmem_wait_ld();
            if (row < args.rows) {
                __nv_bfloat16* dst = args.out + ((size_t)row * args.H + h) * args.ld_out + args.out_col0 + n0 + c0;
#pragma unroll
                for (int j = 0; j < 32; j += 16) {
                    uint32_t o[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) o[q] = pack_bf16(__uint_as_float(r[j + 2 * q]), __uint_as_float(r[j + 2 * q + 1]));
                    if (args.out_v8) {
                        st_global_v8(dst + j, o[0], o[1], o[2], o[3], o[4], o[5], o[6], o[7]);
                    } else {
                        *reinterpret_cast<uint4*>(dst + j) = make_uint4(o[0], o[1], o[2], o[3]);
                        *reinterpret_cast<uint4*>(dst + j + 8) = make_uint4(o[4], o[5], o[6], o[7]);
                    }
                }
            }
        }
    } else if (threadIdx.x == 0) {
        atomicOr(args.status, MLA_STATUS_TIMEOUT);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
    MLA_KT(ROPE ? kKtAbsorb : kKtProject, 2);
}

}  // namespace sm100
}  // namespace mla
