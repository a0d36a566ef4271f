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
    float rope_base;
    int* status;
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
        for (int kc = 0; kc < KCH; ++kc) {
            const int s = kc % STAGES;
            if (kc >= STAGES && !mbar_wait(empty_bar(s), ((kc / STAGES) - 1) & 1)) {
                *abort_flag = 1;
                break;
            }
            const uint32_t a_dst = base + s * C::kStage;
            const uint32_t b_dst = a_dst + C::kABytes;
            mbar_arrive_expect_tx(full_bar(s), C::kStage);
            tma_load_3d(a_dst, &mapA, full_bar(s), kc * 64, h, m0);
            if (B_MN) {
#pragma unroll
                for (int j = 0; j < NT / 64; ++j)
                    tma_load_3d(b_dst + j * 8192, &mapB, full_bar(s), n0 + 64 * j, kc * 64, h);
            } else {
                tma_load_3d(b_dst, &mapB, full_bar(s), kc * 64, n0, h);
            }
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
    __syncwarp();

    // ---------------- epilogue: all four warps, TMEM lane quarter = warp
    const bool ok = mbar_wait(done_bar, 0) && !*abort_flag;
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
                for (int j = 0; j < 32; j += 8) {
                    uint4 v;
                    v.x = pack_bf16(__uint_as_float(r[j + 0]), __uint_as_float(r[j + 1]));
                    v.y = pack_bf16(__uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
                    v.z = pack_bf16(__uint_as_float(r[j + 4]), __uint_as_float(r[j + 5]));
                    v.w = pack_bf16(__uint_as_float(r[j + 6]), __uint_as_float(r[j + 7]));
                    *reinterpret_cast<uint4*>(dst + j) = v;
                }
            }
        }
    } else if (threadIdx.x == 0) {
        atomicOr(args.status, MLA_STATUS_TIMEOUT);
    }
    if (ROPE && blockIdx.y == 0 && row < args.rows) {
        // q_hat[u][h][512 + :] = RoPE(q_rope[u][h], m_u), m_u = seqlens[b] - q_len + i
        const int b = row / args.q_len, i = row % args.q_len;
        const int m = args.seqlens[b] - args.q_len + i;
        const __nv_bfloat16* src = args.q_rope + ((size_t)row * args.H + h) * 64;
        __nv_bfloat16* dst = args.out + ((size_t)row * args.H + h) * args.ld_out + 512;
#pragma unroll 1
        for (int k = 0; k < 32; k += 4) {
            uint4 o;
            uint32_t w[4];
            for (int t = 0; t < 4; ++t) {
                const float x0 = __bfloat162float(src[2 * (k + t)]);
                const float x1 = __bfloat162float(src[2 * (k + t) + 1]);
                float y0, y1;
                mla_rope_pair(x0, x1, k + t, 64, m, args.rope_base, &y0, &y1);
                w[t] = pack_bf16(y0, y1);
            }
            o.x = w[0];
            o.y = w[1];
            o.z = w[2];
            o.w = w[3];
            *reinterpret_cast<uint4*>(dst + 2 * k) = o;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
}

}  // namespace sm100
}  // namespace mla
