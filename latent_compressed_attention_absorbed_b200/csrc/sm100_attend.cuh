// Absorbed-MLA attention in latent space on tcgen05 / TMEM (steps a3 + a4).
//
// For query token (b, i) and all 128 heads at once (the heads are the M
// dimension of a dense contraction against the shared cache):
//   S[h][j]  = scale * ( q_lat[h] . c_KV,j  +  q_rot[h] . k_R,j )     j <= m
//   P        = softmax_j(S)                                          (online)
//   o_lat[h] = sum_j P[h][j] c_KV,j                                   (512-d)
// (092 page, section 二 "缓存压缩也可以做一个代数检查": score the folded query
// against every cached latent, RoPE score added separately; ailearn MLA panel:
// aggregate sum_j p_j c_KV,j before W_UV; m.lsln.cn section 2.1: softmax over
// the whole history.)
//
// Work split.  A CTA owns 64 of the 128 heads of one query token and streams
// full 576-wide cache tiles; the two CTAs of a head pair form one cluster so
// that they run together and each tile is read from HBM once and served to
// the other from L2.  Nothing is exchanged between CTAs.  Per CTA the fp32 accumulator is 64 heads x 512
// latent columns: latent 0..255 lives in TMEM lanes 0..15 of each 32-lane
// subpartition and latent 256..511 in lanes 16..31, both in columns 0..255
// (M = 64 MMAs address either lane half).  Scores are split the same way:
// the lower lane half accumulates S over latent 0..255 + RoPE 0..31, the
// upper half over latent 256..511 + RoPE 32..63, and the two partial sums
// of a row are added with one warp shuffle (lanes t and t+16 hold the same
// head).
//
// Scheduling (split-KV).  The unit of work is a query token (sequence b,
// token i): it attends to keys 0..T_b-q_len+i, cut into 64-key tiles.  The
// clusters divide the concatenated tile list of all units into equal
// contiguous ranges (a fixed per-unit overhead is charged so tiny pieces are
// avoided).  A unit processed by one cluster writes its normalised o_lat
// directly (bf16); a unit cut across clusters writes fp32 partials plus a
// base-2 LSE per head, merged by the combine kernel.
//
// Roles per CTA (192 threads): warp 0 TMA producer, warp 1 TMEM owner and
// MMA issuer, warps 2..5 softmax (warp w reads TMEM subpartition w%4: heads
// 16*(w%4)..+15 in both lane halves).  Every wait is bounded; on expiry the
// kernel flags MLA_STATUS_TIMEOUT, stops issuing work and tears down
// normally.
#pragma once

#include <cuda_bf16.h>
#include <math_constants.h>

#include "mla_rope.cuh"
#include "sm100_ptx.cuh"

namespace mla {
namespace sm100 {

constexpr int kNk = 64;          // keys per tile
constexpr int kHeads = 128;      // heads of a token
constexpr int kRowsCta = 64;     // heads per CTA (M of every MMA)
constexpr int kLat = 512;        // d_c
constexpr int kRope = 64;        // d_r
constexpr int kRow = kLat + kRope;
constexpr int kHalfLat = 256;
constexpr int kHalfRope = 32;

// Shared-memory map (offsets from a 1024-aligned base): a ring of full cache
// tiles, each 9 SW128 chunks of 64 keys x 64 columns (8 latent, 1 RoPE).
constexpr int kChunk = kNk * 128;                          // 8192
constexpr int kTileBytes = 9 * kChunk;                     // 73728
constexpr int kStages = 3;
constexpr int kOffTiles = 0;
constexpr int kOffBars = kOffTiles + kStages * kTileBytes;
constexpr int kAttSmem = kOffBars + 256 + 1024;
// Tensor-memory map: columns of 32 bits; lane half 0 = lanes 0..15 of each
// subpartition, lane half 1 = lanes 16..31 (address lane field + 16).
constexpr int kTmemCols = 512;
constexpr uint32_t kLaneHalf1 = 16u << 16;
constexpr int kTmemO = 0;      // O: half 0 latent 0..255, half 1 latent 256..511 (256 columns)
constexpr int kTmemS = 256;    // S: half 0 partial over K-half a, half 1 over K-half b (64 columns)
constexpr int kTmemP = 320;    // P: 64 bf16 probabilities, two per column, copied in both halves
constexpr int kTmemQ = 352;    // Q-hat: half 0 latent 0..255 + RoPE 0..31, half 1 the rest (144 columns)
constexpr int kAttThreads = 192;

// Barrier indices (8 bytes each) inside the barrier block.
enum {
    kBarFull0 = 0,
    kBarEmpty0 = kBarFull0 + kStages,
    kBarQFull = kBarEmpty0 + kStages,
    kBarSFull,
    kBarSFree,
    kBarPFull,
    kBarPFree,
    kBarOFull,
    kBarOFree,
    kNumBars
};

// Optional timing trace (compile with -DMLA_TRACE): clock64 stamps of the
// first CTA at 16 fixed points of every tile, read back by mla_trace_read.
#ifdef MLA_TRACE
#ifndef MLA_TRACE_CLUSTER
#define MLA_TRACE_CLUSTER 0
#endif
__device__ unsigned long long g_mla_trace[4096][16];
#define MLA_TRACE_POINT(ev, n)                                                                      \
    do {                                                                                            \
        if (cl == MLA_TRACE_CLUSTER && crank == 0 && (n) < 4096) g_mla_trace[(n)][(ev)] = clock64(); \
    } while (0)
#else
#define MLA_TRACE_POINT(ev, n) \
    do {                       \
    } while (0)
#endif

// Scheduling plan written by the plan kernel into the workspace.
struct Plan {
    int L;        // cost units per cluster
    int ovh;      // cost charged per unit (query token)
    int B;        // number of units = sequences x q_len
    int total;    // sum of costs
    int n_split;  // units cut across clusters (listed after the prefix sums)
    int q_len;
    int pad[2];
    // followed by int cost_prefix[B + 1], then int split_unit[B]
};

__device__ __forceinline__ const int* plan_prefix(const Plan* p) { return reinterpret_cast<const int*>(p + 1); }
__device__ __forceinline__ const int* plan_splits(const Plan* p) { return plan_prefix(p) + p->B + 1; }

// Tiles of unit b (0 if its sequence length was invalid).
__device__ __forceinline__ int plan_tiles(const int* pre, int b, int ovh) {
    const int c = pre[b + 1] - pre[b];
    return c > 0 ? c - ovh : 0;
}

// Segment iterator: the (unit, tile range) pieces of cluster `cl`.
struct SegIter {
    const int* pre;
    int B, L, ovh, lo, hi, b;
    __device__ void init(const Plan* plan, int cl) {
        pre = plan_prefix(plan);
        B = plan->B;
        L = plan->L;
        ovh = plan->ovh;
        lo = cl * L;
        hi = lo + L;
        // largest b with pre[b] <= lo
        int a = 0, z = B;
        while (a < z) {
            const int mid = (a + z + 1) / 2;
            if (pre[mid] <= lo) a = mid; else z = mid - 1;
        }
        b = a;
    }
    // Advances to the next non-empty piece; false when done.
    __device__ bool next(int& seq, int& k0, int& k1, bool& whole) {
        while (b < B && pre[b] < hi) {
            const int t = plan_tiles(pre, b, ovh);
            int s = lo - pre[b] - ovh, e = hi - pre[b] - ovh;
            s = s < 0 ? 0 : (s > t ? t : s);
            e = e < 0 ? 0 : (e > t ? t : e);
            const int cur = b++;
            if (e > s) {
                seq = cur;
                k0 = s;
                k1 = e;
                whole = (s == 0 && e == t);
                return true;
            }
        }
        return false;
    }
};

// Flat walk over the tiles of a cluster's pieces, with the piece's bounds.
struct TileWalk {
    SegIter it;
    int seq, k0, k1, t, seg;
    bool whole, valid;
    __device__ void init(const Plan* plan, int cl) {
        it.init(plan, cl);
        seg = 0;
        valid = it.next(seq, k0, k1, whole);
        t = k0;
    }
    __device__ bool first() const { return t == k0; }
    __device__ bool last() const { return t == k1 - 1; }
    __device__ void advance() {
        if (++t >= k1) {
            valid = it.next(seq, k0, k1, whole);
            t = k0;
            ++seg;
        }
    }
};

struct AttendArgs {
    const Plan* plan;
    const int32_t* seqlens;
    int q_len;
    int T_max;
    float scale_log2;             // softmax_scale * log2(e)
    const __nv_bfloat16* q_hat;   // [B][q_len][128][576]
    __nv_bfloat16* o_lat;         // [B][q_len][128][512]
    float* part_o;                // [slots][128 col4][128 heads][4]
    float* part_lse;              // [slots][128]
    int* status;
};

__global__ void __launch_bounds__(kAttThreads, 1)
    mla_attend_kernel(const __grid_constant__ CUtensorMap mapCache, AttendArgs args) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* base_ptr = smem_raw + (base - raw);
    auto bar = [&](int i) { return base + kOffBars + 8u * i; };
    const uint32_t tmem_slot = bar(kNumBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(base_ptr + kOffBars + 8 * (kNumBars + 1));

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const uint32_t crank = cluster_ctarank();
    const int hpart = crank & 1;       // heads 64*hpart .. +63
    const int cl = (int)cluster_id_x();
    const int q_len = args.q_len;
    if (threadIdx.x == 0) MLA_TRACE_POINT(0, 4095);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar(kBarFull0 + s), 1);
            mbar_init(bar(kBarEmpty0 + s), 1);
        }
        mbar_init(bar(kBarQFull), 4);
        mbar_init(bar(kBarSFull), 1);
        mbar_init(bar(kBarSFree), 4);
        mbar_init(bar(kBarPFull), 4);
        mbar_init(bar(kBarPFree), 1);
        mbar_init(bar(kBarOFull), 1);
        mbar_init(bar(kBarOFree), 4);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&mapCache);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(base_ptr + kOffBars + 8 * kNumBars);
    // The set-up above overlaps the previous kernel; the plan, Q-hat and the
    // cache are read only once it has completed.
    if (threadIdx.x == 0) MLA_TRACE_POINT(1, 4095);
    pdl_wait();
    if (threadIdx.x == 0) pdl_trigger();
    if (threadIdx.x == 0) MLA_TRACE_POINT(2, 4095);

    if (warp == 0) {
        // ======================================================== TMA producer (runs up to kStages tiles ahead)
        if (lane == 0) {
            TileWalk w;
            w.init(args.plan, cl);
            for (int n = 0; w.valid && !*abort_flag; ++n, w.advance()) {
                const int st = n % kStages;
                if (n >= kStages && !mbar_wait(bar(kBarEmpty0 + st), ((n / kStages) - 1) & 1)) {
                    *abort_flag = 1;
                    break;
                }
                const uint32_t dst = base + kOffTiles + st * kTileBytes;
                mbar_arrive_expect_tx(bar(kBarFull0 + st), kTileBytes);
                for (int c = 0; c < 9; ++c)
                    tma_load_3d(dst + c * kChunk, &mapCache, bar(kBarFull0 + st), 64 * c, w.t * kNk, w.seq / q_len);
                MLA_TRACE_POINT(0, n);
            }
        }
    } else if (warp == 1) {
        // ======================================================== MMA issuer (whole warp waits, lane 0 issues)
        constexpr uint32_t idS = idesc_bf16_f32(kRowsCta, kNk, false, false);
        constexpr uint32_t idO = idesc_bf16_f32(kRowsCta, kHalfLat, false, true);
        bool ok = true;
        // O(g) += P(g) . C(g) for both latent halves; the first K-step overwrites O at the start of a piece.
        auto issue_O = [&](int g, bool first_in_seg, bool last_in_seg) {
            const uint64_t dO = smem_desc(base + kOffTiles + (g % kStages) * kTileBytes, kChunk, 1024, kSw128);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t acc = (!first_in_seg || k > 0) ? 1u : 0u;
                mma_f16_ts(tmem + kTmemO, tmem + kTmemP + 8 * k, dO + ((2048 * k) >> 4), idO, acc);
                mma_f16_ts(tmem + kLaneHalf1 + kTmemO, tmem + kLaneHalf1 + kTmemP + 8 * k,
                           dO + ((4 * kChunk + 2048 * k) >> 4), idO, acc);
            }
            mma_commit(bar(kBarPFree));
            mma_commit(bar(kBarEmpty0 + (g % kStages)));
            if (last_in_seg) mma_commit(bar(kBarOFull));
        };
        TileWalk w;
        w.init(args.plan, cl);
        bool prev_first = false, prev_last = false, prev_pending = false;
        int prev_seg = 0;
        int g = 0;
        // O(g-1) normally follows S(g) so that S(g) overlaps the softmax of
        // tile g-1; at the end of a piece it goes first, because the softmax
        // warps load the next piece's Q-hat only after that piece's epilogue.
        auto finish_prev = [&]() -> bool {
            if (!mbar_wait(bar(kBarPFull), (g - 1) & 1)) return false;
            if (prev_first && prev_seg > 0 && !mbar_wait(bar(kBarOFree), (prev_seg - 1) & 1)) return false;
            tc_fence_after();
            MLA_TRACE_POINT(4, g - 1);
            if (lane == 0) issue_O(g - 1, prev_first, prev_last);
            __syncwarp();
            MLA_TRACE_POINT(5, g - 1);
            prev_pending = false;
            return true;
        };
        // Descriptor templates: start-address field (bits 0..13, address >> 4)
        // is advanced by adding byte offsets >> 4 to one base descriptor.
        const uint64_t dS0 = smem_desc(base + kOffTiles, 16, 1024, kSw128);
        const uint64_t dO0 = smem_desc(base + kOffTiles, kChunk, 1024, kSw128);
        int T_b = 0;
        for (; w.valid && ok && !*abort_flag; ++g, w.advance()) {
            if (prev_pending && prev_last && !finish_prev()) { ok = false; break; }
            if (w.first()) {
                T_b = args.seqlens[w.seq / q_len];
                if (!mbar_wait(bar(kBarQFull), w.seg & 1)) { ok = false; break; }
            }
            const int st = g % kStages;
            const uint32_t tile_off = kOffTiles + st * kTileBytes;
            const uint32_t tile = base + tile_off;
            if (!mbar_wait(bar(kBarFull0 + st), (g / kStages) & 1)) { ok = false; break; }
            MLA_TRACE_POINT(1, g);
            const int valid = T_b - w.t * kNk;
            if (valid < kNk) {
                // Rows at or beyond T_b hold no cached token: zero them so that
                // masked (p = 0) rows cannot inject NaN/Inf into P.C.
                const int r0 = valid < 0 ? 0 : valid;
                for (int r = r0 + (lane >> 3); r < kNk; r += 4)
                    for (int c = 0; c < 9; ++c) st_shared_v4(tile + c * kChunk + r * 128 + (lane & 7) * 16, 0, 0, 0, 0);
                fence_proxy_async_smem();
            }
            __syncwarp();
            // S(g) reuses the S columns: the softmax warps must have read S(g-1).
            if (g > 0 && !mbar_wait(bar(kBarSFree), (g - 1) & 1)) { ok = false; break; }
            tc_fence_after();
            MLA_TRACE_POINT(2, g);
            if (lane == 0) {
                // half a: latent chunks 0..3 then RoPE columns 0..31; half b: chunks 4..7 then RoPE 32..63
                const uint64_t dS = dS0 + ((tile_off) >> 4);
#pragma unroll
                for (int kk = 0; kk < 18; ++kk) {
                    const uint32_t oa = kk < 16 ? (kk / 4) * kChunk + 32 * (kk % 4) : 8 * kChunk + 32 * (kk - 16);
                    const uint32_t ob = kk < 16 ? (4 + kk / 4) * kChunk + 32 * (kk % 4) : 8 * kChunk + 64 + 32 * (kk - 16);
                    mma_f16_ts(tmem + kTmemS, tmem + kTmemQ + 8 * kk, dS + (oa >> 4), idS, kk ? 1u : 0u);
                    mma_f16_ts(tmem + kLaneHalf1 + kTmemS, tmem + kLaneHalf1 + kTmemQ + 8 * kk, dS + (ob >> 4), idS,
                               kk ? 1u : 0u);
                }
                mma_commit(bar(kBarSFull));
            }
            __syncwarp();
            MLA_TRACE_POINT(3, g);
            if (prev_pending && !finish_prev()) { ok = false; break; }
            prev_first = w.first();
            prev_last = w.last();
            prev_seg = w.seg;
            prev_pending = true;
        }
        if (ok && !*abort_flag && prev_pending && !finish_prev()) ok = false;
        if (!ok) *abort_flag = 1;
    } else {
        // ======================================================== softmax warps 2..5
        // Thread (quarter, lane): head row m = 16*quarter + lane%16 of this CTA,
        // lane half lh = lane/16: it reads the lh partial scores, handles keys
        // 32*lh..32*lh+31 of the row, and owns latent half lh of O.
        const int quarter = warp & 3;
        const int lh = lane >> 4;
        const int m = quarter * 16 + (lane & 15);
        const int head = hpart * kRowsCta + m;
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;  // the warp's subpartition
        const float sl2 = args.scale_log2;
        bool ok = true;
        TileWalk w;
        w.init(args.plan, cl);
        float m_used = -CUDART_INF_F, l_sum = 0.f;
        int n_keys = 0;
        for (int g = 0; w.valid && ok && !*abort_flag; ++g, w.advance()) {
            if (w.first()) {
                // Q-hat row `head`, K-half lh -> TMEM (S(g-1), the last reader of the old Q-hat, has completed).
                const int u = w.seq;
                const uint4* src = reinterpret_cast<const uint4*>(args.q_hat + ((size_t)u * kHeads + head) * kRow);
                // 36 loads of 16 bytes in two batches (latent 0..127 | latent 128..255 + RoPE)
                {
                    uint4 x[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) x[j] = __ldg(src + lh * 32 + j);
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        uint32_t v[32];
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            v[4 * j] = x[8 * c + j].x; v[4 * j + 1] = x[8 * c + j].y;
                            v[4 * j + 2] = x[8 * c + j].z; v[4 * j + 3] = x[8 * c + j].w;
                        }
                        tmem_st32(tmem + lane_addr + kTmemQ + 32 * c, v);
                    }
                }
                {
                    uint4 x[20];
#pragma unroll
                    for (int j = 0; j < 16; ++j) x[j] = __ldg(src + lh * 32 + 16 + j);
#pragma unroll
                    for (int j = 0; j < 4; ++j) x[16 + j] = __ldg(src + 64 + lh * 4 + j);
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        uint32_t v[32];
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            v[4 * j] = x[8 * c + j].x; v[4 * j + 1] = x[8 * c + j].y;
                            v[4 * j + 2] = x[8 * c + j].z; v[4 * j + 3] = x[8 * c + j].w;
                        }
                        tmem_st32(tmem + lane_addr + kTmemQ + 64 + 32 * c, v);
                    }
                    uint32_t v[16];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        v[4 * j] = x[16 + j].x; v[4 * j + 1] = x[16 + j].y;
                        v[4 * j + 2] = x[16 + j].z; v[4 * j + 3] = x[16 + j].w;
                    }
                    tmem_st16(tmem + lane_addr + kTmemQ + 128, v);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kBarQFull));
                if (threadIdx.x == 64) MLA_TRACE_POINT(7, 4095);
            }
            // ---- partial S(g) of this lane half
            if (!mbar_wait(bar(kBarSFull), g & 1)) { ok = false; break; }
            tc_fence_after();
            MLA_TRACE_POINT(7, g);
            uint32_t va[32], vb[32];
            tmem_ld32(tmem + lane_addr + kTmemS, va);
            tmem_ld32(tmem + lane_addr + kTmemS + 32, vb);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kBarSFree));
            // ---- full scores of keys 32*lh .. +31: own partial + the other half's (lane ^ 16)
            float s[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float give = __uint_as_float(lh ? va[j] : vb[j]);  // the half the partner scores
                const float mine = __uint_as_float(lh ? vb[j] : va[j]);
                const float other = __shfl_xor_sync(0xffffffffu, give, 16);
                s[j] = (mine + other) * sl2;
            }
            // unit u = (b, i) sees keys 0..T_b-q_len+i
            if (w.first()) n_keys = args.seqlens[w.seq / q_len] - q_len + 1 + w.seq % q_len;
            const int key0 = w.t * kNk + 32 * lh;
            if (key0 + 32 > n_keys) {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (key0 + j >= n_keys) s[j] = -CUDART_INF_F;
            }
            float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
            for (int j = 4; j < 32; j += 4) {
                mx0 = fmaxf(mx0, s[j]); mx1 = fmaxf(mx1, s[j + 1]);
                mx2 = fmaxf(mx2, s[j + 2]); mx3 = fmaxf(mx3, s[j + 3]);
            }
            float mx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            const bool first = w.first();
            const bool grow = mx > m_used + 8.0f;  // rescale only when the max grows by > 2^8
            const float mb_new = grow ? mx : m_used;
            const float mb = (mb_new == -CUDART_INF_F) ? 0.f : mb_new;
            uint32_t own[16];
            float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float p0 = ex2(s[2 * j] - mb), p1 = ex2(s[2 * j + 1] - mb);
                rs0 += p0;
                rs1 += p1;
                own[j] = pack_bf16(p0, p1);
            }
            float rs = rs0 + rs1;
            rs += __shfl_xor_sync(0xffffffffu, rs, 16);
            uint32_t pk[32];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const uint32_t oth = __shfl_xor_sync(0xffffffffu, own[j], 16);
                pk[j] = lh ? oth : own[j];
                pk[16 + j] = lh ? own[j] : oth;
            }
            MLA_TRACE_POINT(11, g);
            // P(g) overwrites P(g-1) and a rescale touches O: wait for O += P(g-1) C(g-1).
            if (g > 0 && !mbar_wait(bar(kBarPFree), (g - 1) & 1)) { ok = false; break; }
            tc_fence_after();
            MLA_TRACE_POINT(12, g);
            if (grow) {
                if (!first) {
                    const float f = ex2(m_used - mx);
                    l_sum *= f;
#pragma unroll 1
                    for (int c0 = 0; c0 < kHalfLat; c0 += 32) {
                        uint32_t v[32];
                        tmem_ld32(tmem + lane_addr + kTmemO + c0, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * f);
                        tmem_st32(tmem + lane_addr + kTmemO + c0, v);
                    }
                }
                m_used = mx;
            }
            l_sum += rs;
            tmem_st32(tmem + lane_addr + kTmemP, pk);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kBarPFull));
            MLA_TRACE_POINT(13, g);
            // ---- epilogue at the end of a piece: this thread owns O row m, latent half lh
            if (w.last()) {
                if (!mbar_wait(bar(kBarOFull), w.seg & 1)) { ok = false; break; }
                tc_fence_after();
                if (threadIdx.x == 64) MLA_TRACE_POINT(5, 4095);
                const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
                const int u = w.seq;
                if (w.whole) {
                    __nv_bfloat16* dst = args.o_lat + ((size_t)u * kHeads + head) * kLat + lh * kHalfLat;
#pragma unroll 1
                    for (int c0 = 0; c0 < kHalfLat; c0 += 32) {
                        uint32_t v[32];
                        tmem_ld32(tmem + lane_addr + kTmemO + c0, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 32; j += 8) {
                            uint4 o;
                            o.x = pack_bf16(__uint_as_float(v[j]) * inv, __uint_as_float(v[j + 1]) * inv);
                            o.y = pack_bf16(__uint_as_float(v[j + 2]) * inv, __uint_as_float(v[j + 3]) * inv);
                            o.z = pack_bf16(__uint_as_float(v[j + 4]) * inv, __uint_as_float(v[j + 5]) * inv);
                            o.w = pack_bf16(__uint_as_float(v[j + 6]) * inv, __uint_as_float(v[j + 7]) * inv);
                            *reinterpret_cast<uint4*>(dst + c0 + j) = o;
                        }
                    }
                } else {
                    // fp32 partial, head-minor: [slot][col4][head][4] so that the 16 lanes of
                    // a half warp (16 consecutive heads) write 256 contiguous bytes per store.
                    const int slot = cl + u;
                    float4* dst = reinterpret_cast<float4*>(args.part_o) + (size_t)slot * (kLat / 4) * kHeads + head;
#pragma unroll 1
                    for (int c0 = 0; c0 < kHalfLat; c0 += 32) {
                        uint32_t v[32];
                        tmem_ld32(tmem + lane_addr + kTmemO + c0, v);
                        tmem_wait_ld();
                        const int k0 = (lh * kHalfLat + c0) / 4;
#pragma unroll
                        for (int j = 0; j < 32; j += 4)
                            dst[(size_t)(k0 + j / 4) * kHeads] =
                                make_float4(__uint_as_float(v[j]) * inv, __uint_as_float(v[j + 1]) * inv,
                                            __uint_as_float(v[j + 2]) * inv, __uint_as_float(v[j + 3]) * inv);
                    }
                    if (lh == 0)
                        args.part_lse[(size_t)slot * kHeads + head] =
                            l_sum > 0.f ? m_used + __log2f(l_sum) : -CUDART_INF_F;
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kBarOFree));
                if (threadIdx.x == 64) MLA_TRACE_POINT(6, 4095);
                m_used = -CUDART_INF_F;
                l_sum = 0.f;
            }
        }
        if (!ok) *abort_flag = 1;
    }

    if (*abort_flag && threadIdx.x == 0) atomicOr(args.status, MLA_STATUS_TIMEOUT);
    if (threadIdx.x == 64) MLA_TRACE_POINT(3, 4095);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, kTmemCols);
    if (threadIdx.x == 32) MLA_TRACE_POINT(4, 4095);
}

// ------------------------------------------------------------------ plan

// cost_b = ceil(T_b / 64) + ovh (0 for an invalid length); prefix sums and the
// per-cluster share L = ceil(total / clusters), at least min_units; the list
// of sequences cut across clusters; o_lat = 0 for sequences with an invalid
// length (their decode has no defined result).  One warp.
__device__ __forceinline__ void mla_plan_warp(const int32_t* __restrict__ seqlens, int B, int q_len, int T_max,
                                              int clusters, int ovh, int min_units, Plan* plan, int* status,
                                              __nv_bfloat16* o_lat, int lane) {
    const int U = B * q_len;
    int* pre = reinterpret_cast<int*>(plan + 1);
    int* splits = pre + U + 1;
    int carry = 0;
    if (lane == 0) pre[0] = 0;
    for (int base = 0; base < U; base += 32) {
        const int u = base + lane;
        int c = 0;
        if (u < U) {
            const int T = seqlens[u / q_len];
            if (T < q_len || T > T_max) {
                if (u % q_len == 0) atomicOr(status, MLA_STATUS_BAD_SEQLEN);
            } else {
                c = (T - q_len + 1 + u % q_len + kNk - 1) / kNk + ovh;
            }
        }
        int v = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += y;
        }
        if (u < U) pre[u + 1] = carry + v;
        carry += __shfl_sync(0xffffffffu, v, 31);
    }
    int L = (carry + clusters - 1) / clusters;
    if (L < min_units) L = min_units;
    if (L < 1) L = 1;
    __syncwarp();
    int n_split = 0;
    for (int base = 0; base < U; base += 32) {
        const int u = base + lane;
        bool split = false, invalid = false;
        if (u < U) {
            const int lo = pre[u], hi = pre[u + 1];
            if (hi == lo) invalid = true;
            else split = (lo + ovh) / L != (hi - 1) / L;
        }
        const unsigned m = __ballot_sync(0xffffffffu, split);
        if (split) splits[n_split + __popc(m & ((1u << lane) - 1))] = u;
        n_split += __popc(m);
        unsigned inv = __ballot_sync(0xffffffffu, invalid);
        while (inv) {
            const int ui = base + __ffs(inv) - 1;
            inv &= inv - 1;
            uint4* dst = reinterpret_cast<uint4*>(o_lat + (size_t)ui * kHeads * kLat);
            for (int i = lane; i < kHeads * kLat / 8; i += 32) dst[i] = make_uint4(0, 0, 0, 0);
        }
    }
    if (lane == 0) {
        plan->L = L;
        plan->ovh = ovh;
        plan->B = U;
        plan->total = carry;
        plan->n_split = n_split;
        plan->q_len = q_len;
    }
}

__global__ void __launch_bounds__(32) mla_plan_kernel(const int32_t* __restrict__ seqlens, int B, int q_len,
                                                      int T_max, int clusters, int ovh, int min_units, Plan* plan,
                                                      int* status, __nv_bfloat16* o_lat) {
    mla_plan_warp(seqlens, B, q_len, T_max, clusters, ovh, min_units, plan, status, o_lat, threadIdx.x);
}

// ------------------------------------------------------------------ combine

// Merge of split partials: o_lat = sum_s 2^(lse_s - M) o_s / sum_s 2^(lse_s - M)
// with M = max_s lse_s (the softmax of the pieces' log-sum-exps).
//
// One thread per (split unit, 4 latent columns, head, piece group): the 128
// consecutive threads of a group read the 128 heads of one column quad, a
// contiguous 2 KiB of the head-minor partials.  A CTA covers KPC column
// quads; its G groups take every G-th piece and keep a running (max, sum,
// accumulator) each, merged through shared memory at the end.  G = 1 suits
// batches whose units are cut into a few pieces; G = 8 gives small batches
// (a unit cut into tens of pieces) enough loads in flight.
template <int G, int KPC>
__global__ void __launch_bounds__(128 * G * KPC) mla_combine_kernel(const Plan* __restrict__ plan,
                                                                    const float* __restrict__ part_o,
                                                                    const float* __restrict__ part_lse,
                                                                    __nv_bfloat16* __restrict__ o_lat) {
    constexpr int kPerUnit = (kLat / 4) / KPC;  // CTAs per split unit
    constexpr int kBatch = 4;                   // pieces whose loads are issued together
    __shared__ float4 s_acc[G > 1 ? G : 1][KPC][kHeads];
    __shared__ float2 s_mw[G > 1 ? G : 1][KPC][kHeads];
    pdl_wait();
    pdl_trigger();
    const int work = blockIdx.x / kPerUnit;
    if (work >= plan->n_split) return;
    const int h = threadIdx.x % kHeads;
    const int kk = (threadIdx.x / kHeads) % KPC;
    const int g = threadIdx.x / (kHeads * KPC);
    const int k = (blockIdx.x % kPerUnit) * KPC + kk;  // column quad
    const int u = plan_splits(plan)[work];
    const int* pre = plan_prefix(plan);
    const int L = plan->L, ovh = plan->ovh;
    const int tiles = plan_tiles(pre, u, ovh);
    const int c_lo = pre[u], c_hi = pre[u + 1];
    const int p_lo = c_lo / L, p_hi = (c_hi - 1) / L;
    // Cluster p holds tiles [p L - c_lo - ovh, (p+1) L - c_lo - ovh) of the
    // unit, clipped to [0, tiles); an empty clip wrote no partial.
    auto nonempty = [&](int p) {
        int s0 = p * L - c_lo - ovh, e0 = (p + 1) * L - c_lo - ovh;
        s0 = s0 < 0 ? 0 : (s0 > tiles ? tiles : s0);
        e0 = e0 < 0 ? 0 : (e0 > tiles ? tiles : e0);
        return e0 > s0;
    };
    const float4* po = reinterpret_cast<const float4*>(part_o) + (size_t)k * kHeads + h;
    float m = -CUDART_INF_F, wsum = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int p0 = p_lo + g; p0 <= p_hi; p0 += G * kBatch) {
        float lse[kBatch];
        float4 v[kBatch];
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
            const int p = p0 + j * G;
            lse[j] = -CUDART_INF_F;
            v[j] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (p <= p_hi && nonempty(p)) {
                const size_t slot = (size_t)(p + u);
                lse[j] = __ldg(part_lse + slot * kHeads + h);
                v[j] = __ldg(po + slot * (kLat / 4) * kHeads);
            }
        }
        float mb = m;
#pragma unroll
        for (int j = 0; j < kBatch; ++j) mb = fmaxf(mb, lse[j]);
        if (mb == -CUDART_INF_F) continue;  // nothing but empty pieces so far
        const float r = exp2f(m - mb);      // m = -inf gives 0
        wsum *= r;
        acc.x *= r;
        acc.y *= r;
        acc.z *= r;
        acc.w *= r;
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
            const float w = exp2f(lse[j] - mb);  // empty piece: 2^-inf = 0
            wsum += w;
            acc.x += w * v[j].x;
            acc.y += w * v[j].y;
            acc.z += w * v[j].z;
            acc.w += w * v[j].w;
        }
        m = mb;
    }
    if constexpr (G > 1) {
        s_acc[g][kk][h] = acc;
        s_mw[g][kk][h] = make_float2(m, wsum);
        __syncthreads();
        if (g != 0) return;
        for (int j = 1; j < G; ++j) {
            const float2 mw = s_mw[j][kk][h];
            const float mb = fmaxf(m, mw.x);
            if (mb == -CUDART_INF_F) continue;
            const float r0 = exp2f(m - mb), r1 = exp2f(mw.x - mb);
            const float4 a1 = s_acc[j][kk][h];
            wsum = wsum * r0 + mw.y * r1;
            acc.x = acc.x * r0 + a1.x * r1;
            acc.y = acc.y * r0 + a1.y * r1;
            acc.z = acc.z * r0 + a1.z * r1;
            acc.w = acc.w * r0 + a1.w * r1;
            m = mb;
        }
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    uint2 o;
    o.x = pack_bf16(acc.x * inv, acc.y * inv);
    o.y = pack_bf16(acc.z * inv, acc.w * inv);
    *reinterpret_cast<uint2*>(o_lat + ((size_t)u * kHeads + h) * kLat + 4 * k) = o;
}

}  // namespace sm100
}  // namespace mla
