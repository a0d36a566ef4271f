// Dense bf16 projections around the attention step, on tcgen05 / TMEM.
//
//   Y[m][n] = sum_k A[m][k] B[n][k]     A: [rows][K] activations, B: [N][K]
//                                        weights (the row-major layout of a
//                                        linear layer), both K contiguous.
//
// Two projections of the MLA block use it:
//   * the cache append from the block input x (hidden 7168): [c_KV || k_R]
//     = [W_DKV; W_KR] x, N = 576, K = 7168 (m.lsln.cn/news/222502 section 2.2:
//     c^KV = W^DKV h; 092 page, section 二);
//   * the output projection after W_UV: y = W_O out, N = 7168 (hidden),
//     K = H * d_v = 16384 (ailearn.mscapital.top MLA panel: Sigma p c_KV,
//     then W_UV and the output projection).
// At decode sizes (a few hundred query tokens) both are bound by the weight
// read, so the grid splits K as well as N: S splits x (N / NT) column tiles
// x (rows / 128) row tiles of CTAs stream disjoint slices of the weights.
// Each CTA accumulates a 128 x NT fp32 tile in TMEM (M = 128 MMAs, K = 16)
// from a TMA ring of 64-wide K chunks and stores it: as fp32 partials
// P[s][m][n] when S > 1 (a finishing kernel adds the S partials in a fixed
// order), or as bf16 Y directly when S = 1.
//
// Roles (128 threads): warp 0 lane 0 issues TMA loads (the weight tiles of
// the first stages before the grid-dependency wait: weights are never
// written by the kernel that precedes this one); warp 1 owns TMEM and
// lane 0 issues the MMAs; all four warps drain TMEM (lane quarter = warp).
// Every barrier wait is bounded; on expiry the CTA flags MLA_STATUS_TIMEOUT
// and skips its store.
#pragma once

#include <cuda_bf16.h>

#include "mla.h"
#include "sm100_ptx.cuh"

namespace mla {
namespace sm100 {

template <int NT, int STAGES>
struct LinCfg {
    static constexpr int kABytes = 128 * 128;  // 128 rows x 64 bf16 (the A box may hold fewer rows)
    static constexpr int kBBytes = NT * 128;   // NT rows x 64 bf16
    static constexpr int kStage = kABytes + kBBytes;
    static constexpr int kSmem = STAGES * kStage + 256 + 1024;
    static constexpr int kTmemCols = NT < 32 ? 32 : NT;
    static constexpr uint32_t kIdesc = idesc_bf16_f32(128, NT, false, false);
    static_assert(NT % 32 == 0 && NT >= 32 && NT <= 256, "column tile");
};

struct LinArgs {
    int rows;            // M extent
    int N;               // output columns
    int kc_per_split;    // 64-wide K chunks per split
    int kc_total;        // K / 64
    int a_rows;          // rows of each A box (multiple of 16, <= 128)
    float* part;         // if set: [S][rows][N] fp32 partials
    __nv_bfloat16* out;  // otherwise (S = 1): [rows][N] bf16
    int* status;
    uint64_t wait_limit_ns;
};

// mapA: A as 2-D [rows][K], box 64 x a_rows, SW128.  mapB: B as [N][K], box 64 x NT, SW128.
template <int NT, int STAGES>
__global__ void __launch_bounds__(128, 1)
    linear_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB, LinArgs args) {
    using C = LinCfg<NT, STAGES>;
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
    const uint64_t lim = args.wait_limit_ns;

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int n0 = blockIdx.x * NT;
    const int split = blockIdx.y;
    const int m0 = blockIdx.z * 128;
    const int kc0 = split * args.kc_per_split;
    const int kc1 = min(kc0 + args.kc_per_split, args.kc_total);
    const int nk = kc1 > kc0 ? kc1 - kc0 : 0;

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
    const uint32_t tx = (uint32_t)args.a_rows * 128 + C::kBBytes;
    int n_loads = 0;

    if (warp == 0 && lane == 0) {
        // ---------------- producer
        const int pre = nk < STAGES ? nk : STAGES;
        for (int i = 0; i < pre; ++i) {
            mbar_arrive_expect_tx(full_bar(i), tx);
            tma_load_2d(base + i * C::kStage + C::kABytes, &mapB, full_bar(i), (kc0 + i) * 64, n0);
        }
        pdl_wait();
        pdl_trigger();
        for (int i = 0; i < nk; ++i) {
            const int s = i % STAGES;
            if (i >= pre) {
                if (!mbar_wait(empty_bar(s), ((i / STAGES) - 1) & 1, lim)) {
                    *abort_flag = 1;
                    break;
                }
                mbar_arrive_expect_tx(full_bar(s), tx);
                tma_load_2d(base + s * C::kStage + C::kABytes, &mapB, full_bar(s), (kc0 + i) * 64, n0);
            }
            tma_load_2d(base + s * C::kStage, &mapA, full_bar(s), (kc0 + i) * 64, m0);
            n_loads = i + 1;
        }
        // Loads issued before the wait whose A half was never issued (an
        // early stop) would leave their stage waiting for bytes: none can
        // exist, since the loop issues the A half of every pre-issued stage
        // before it can stop (a stop happens only at i >= pre).
    }
    if (warp == 1 && lane == 0) {
        // ---------------- MMA issuer
        for (int i = 0; i < nk; ++i) {
            const int s = i % STAGES;
            if (*abort_flag || !mbar_wait(full_bar(s), (i / STAGES) & 1, lim)) {
                *abort_flag = 1;
                break;
            }
            tc_fence_after();
            const uint32_t a_addr = base + s * C::kStage;
            const uint32_t b_addr = a_addr + C::kABytes;
#pragma unroll
            for (int k = 0; k < 4; ++k)
                mma_f16_ss(tmem, smem_desc(a_addr + 32 * k, 16, 1024, kSw128), smem_desc(b_addr + 32 * k, 16, 1024, kSw128),
                           C::kIdesc, (i | k) ? 1u : 0u);
            mma_commit(empty_bar(s));
        }
        mma_commit(done_bar);
    }
    // The other lanes of the producer and MMA warps wait here for their lane 0
    // (a warp barrier: they must not spin on the completion barrier below
    // while lane 0 of the same warp runs its loop).
    __syncwarp();
    pdl_wait();  // nothing is written before the kernels this one depends on have completed
    // ---------------- epilogue: all four warps, TMEM lane quarter = warp
    const bool ok = __all_sync(0xffffffffu, mbar_wait(done_bar, 0, lim) && !*abort_flag) && nk > 0;
    tc_fence_after();
    const int row = m0 + warp * 32 + lane;
    if (ok) {
#pragma unroll 1
        for (int c0 = 0; c0 < NT; c0 += 32) {
            uint32_t r[32];
            tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + c0, r);
            tmem_wait_ld();
            if (row < args.rows) {
                if (args.part) {
                    float* dst = args.part + ((size_t)split * args.rows + row) * args.N + n0 + c0;
#pragma unroll
                    for (int j = 0; j < 32; j += 8)
                        st_global_v8(dst + j, r[j], r[j + 1], r[j + 2], r[j + 3], r[j + 4], r[j + 5], r[j + 6], r[j + 7]);
                } else {
                    __nv_bfloat16* dst = args.out + (size_t)row * args.N + n0 + c0;
#pragma unroll
                    for (int j = 0; j < 32; j += 16) {
                        uint32_t o[8];
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            o[q] = pack_bf16(__uint_as_float(r[j + 2 * q]), __uint_as_float(r[j + 2 * q + 1]));
                        st_global_v8(dst + j, o[0], o[1], o[2], o[3], o[4], o[5], o[6], o[7]);
                    }
                }
            }
        }
    } else if (threadIdx.x == 0 && nk > 0) {
        atomicOr(args.status, MLA_STATUS_TIMEOUT);
    }
    // Drain: stage loads still in flight after an early stop.
    if (warp == 0 && lane == 0 && *abort_flag)
        for (int i = n_loads > STAGES ? n_loads - STAGES : 0; i < n_loads; ++i)
            mbar_wait(full_bar(i % STAGES), (i / STAGES) & 1, lim);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
}

}  // namespace sm100
}  // namespace mla
