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
// full 576-wide cache tiles; the two CTAs of a head pair (and the q_len
// token groups) form one cluster so that they run together and each tile is
// read from HBM once and served to the others from L2.  Nothing is
// exchanged between CTAs.  Per CTA the fp32 accumulator is 64 heads x 512
// latent columns: latent 0..255 lives in TMEM lanes 0..15 of each 32-lane
// subpartition and latent 256..511 in lanes 16..31, both in columns 0..255
// (M = 64 MMAs address either lane half).  Scores are split the same way:
// the lower lane half accumulates S over latent 0..255 + RoPE 0..31, the
// upper half over latent 256..511 + RoPE 32..63, and the two partial sums
// of a row are added with one warp shuffle (lanes t and t+16 hold the same
// head).
//
// Scheduling (split-KV).  Sequences are cut into 64-key tiles; the clusters
// divide the concatenated tile list into equal contiguous ranges (a fixed
// per-sequence overhead is charged so tiny pieces are avoided).  A sequence
// processed by one cluster writes its normalised o_lat directly (bf16); a
// sequence cut across clusters writes fp32 partials plus a base-2 LSE per
// head, merged by the combine kernel.
//
// Roles per CTA (192 threads): warp 0 TMA producer, warp 1 TMEM owner and
// MMA issuer, warps 2..5 softmax (warp w reads TMEM subpartition w%4: heads
// 16*(w%4)..+15 in both lane halves).  Every wait is bounded; on expiry the
// kernel flags MLA_STATUS_TIMEOUT, stops issuing work and tears down
// normally.
#pragma once

#include <cuda_bf16.h>
#include <math_constants.h>

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
__device__ unsigned long long g_mla_trace[4096][16];
#define MLA_TRACE_POINT(ev, n)                                                 \
    do {                                                                       \
        if (cl == 0 && crank == 0 && (n) < 4096) g_mla_trace[(n)][(ev)] = clock64(); \
    } while (0)
#else
#define MLA_TRACE_POINT(ev, n) \
    do {                       \
    } while (0)
#endif

// Scheduling plan written by the plan kernel into the workspace.
struct Plan {
    int L;       // cost units per cluster
    int ovh;     // cost charged per sequence
    int B;
    int total;   // sum of costs
    // followed by int cost_prefix[B + 1]
};

__device__ __forceinline__ const int* plan_prefix(const Plan* p) { return reinterpret_cast<const int*>(p + 1); }

// Tiles of sequence b (0 if its length was invalid).
__device__ __forceinline__ int plan_tiles(const int* pre, int b, int ovh) {
    const int c = pre[b + 1] - pre[b];
    return c > 0 ? c - ovh : 0;
}

// Segment iterator: the (sequence, tile range) pieces of cluster `cl`.
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
    float* part_o;                // [slots][q_len][128][512]
    float* part_lse;              // [slots][q_len][128]
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
    const int qi = crank >> 1;         // query token of this CTA
    const int cl = (int)cluster_id_x();
    const int q_len = args.q_len;

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
                    tma_load_3d(dst + c * kChunk, &mapCache, bar(kBarFull0 + st), 64 * c, w.t * kNk, w.seq);
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
            const uint32_t tile = base + kOffTiles + (g % kStages) * kTileBytes;
            for (int k = 0; k < 4; ++k) {
                const uint32_t acc = (!first_in_seg || k > 0) ? 1u : 0u;
                mma_f16_ts(tmem + kTmemO, tmem + kTmemP + 8 * k, smem_desc(tile + 2048 * k, kChunk, 1024, kSw128),
                           idO, acc);
                mma_f16_ts(tmem + kLaneHalf1 + kTmemO, tmem + kLaneHalf1 + kTmemP + 8 * k,
                           smem_desc(tile + 4 * kChunk + 2048 * k, kChunk, 1024, kSw128), idO, acc);
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
        for (; w.valid && ok && !*abort_flag; ++g, w.advance()) {
            if (prev_pending && prev_last && !finish_prev()) { ok = false; break; }
            const int T_b = args.seqlens[w.seq];
            if (w.first() && !mbar_wait(bar(kBarQFull), w.seg & 1)) { ok = false; break; }
            const int st = g % kStages;
            const uint32_t tile = base + kOffTiles + st * kTileBytes;
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
                for (int kk = 0; kk < 18; ++kk) {
                    const int ca = kk < 16 ? kk / 4 : 8, cb = kk < 16 ? 4 + kk / 4 : 8;
                    const int oa = kk < 16 ? 32 * (kk % 4) : 32 * (kk - 16);
                    const int ob = kk < 16 ? 32 * (kk % 4) : 64 + 32 * (kk - 16);
                    mma_f16_ts(tmem + kTmemS, tmem + kTmemQ + 8 * kk,
                               smem_desc(tile + ca * kChunk + oa, 16, 1024, kSw128), idS, kk ? 1u : 0u);
                    mma_f16_ts(tmem + kLaneHalf1 + kTmemS, tmem + kLaneHalf1 + kTmemQ + 8 * kk,
                               smem_desc(tile + cb * kChunk + ob, 16, 1024, kSw128), idS, kk ? 1u : 0u);
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
        for (int g = 0; w.valid && ok && !*abort_flag; ++g, w.advance()) {
            if (w.first()) {
                // Q-hat row `head`, K-half lh -> TMEM (S(g-1), the last reader of the old Q-hat, has completed).
                const int u = w.seq * q_len + qi;
                const uint4* src = reinterpret_cast<const uint4*>(args.q_hat + ((size_t)u * kHeads + head) * kRow);
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t v[32];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint4 x = __ldg(src + lh * 32 + c * 8 + j);
                        v[4 * j] = x.x; v[4 * j + 1] = x.y; v[4 * j + 2] = x.z; v[4 * j + 3] = x.w;
                    }
                    tmem_st32(tmem + lane_addr + kTmemQ + 32 * c, v);
                }
                uint32_t v[16];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint4 x = __ldg(src + 64 + lh * 4 + j);
                    v[4 * j] = x.x; v[4 * j + 1] = x.y; v[4 * j + 2] = x.z; v[4 * j + 3] = x.w;
                }
                tmem_st16(tmem + lane_addr + kTmemQ + 128, v);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kBarQFull));
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
            const int T_b = args.seqlens[w.seq];
            const int n_keys = T_b - q_len + 1 + qi;  // query qi attends to keys 0..n_keys-1
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
                const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
                const int u = w.seq * q_len + qi;
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
                    const int slot = cl + w.seq;
                    float* dst = args.part_o + (((size_t)slot * q_len + qi) * kHeads + head) * kLat + lh * kHalfLat;
#pragma unroll 1
                    for (int c0 = 0; c0 < kHalfLat; c0 += 32) {
                        uint32_t v[32];
                        tmem_ld32(tmem + lane_addr + kTmemO + c0, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 32; j += 4) {
                            float4 o = make_float4(__uint_as_float(v[j]) * inv, __uint_as_float(v[j + 1]) * inv,
                                                   __uint_as_float(v[j + 2]) * inv, __uint_as_float(v[j + 3]) * inv);
                            *reinterpret_cast<float4*>(dst + c0 + j) = o;
                        }
                    }
                    if (lh == 0)
                        args.part_lse[((size_t)slot * q_len + qi) * kHeads + head] =
                            l_sum > 0.f ? m_used + __log2f(l_sum) : -CUDART_INF_F;
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kBarOFree));
                m_used = -CUDART_INF_F;
                l_sum = 0.f;
            }
        }
        if (!ok) *abort_flag = 1;
    }

    if (*abort_flag && threadIdx.x == 0) atomicOr(args.status, MLA_STATUS_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------------ plan

// cost_b = ceil(T_b / 64) + ovh (0 for an invalid length); prefix sums and the
// per-cluster share L = ceil(total / clusters), at least min_units.
__global__ void mla_plan_kernel(const int32_t* __restrict__ seqlens, int B, int q_len, int T_max, int clusters,
                                int ovh, int min_units, Plan* plan, int* status) {
    __shared__ int warp_sums[32];
    __shared__ int carry;
    int* pre = reinterpret_cast<int*>(plan + 1);
    if (threadIdx.x == 0) {
        carry = 0;
        pre[0] = 0;
    }
    __syncthreads();
    for (int base = 0; base < B; base += blockDim.x) {
        const int b = base + threadIdx.x;
        int c = 0;
        if (b < B) {
            const int T = seqlens[b];
            if (T < q_len || T > T_max) atomicOr(status, MLA_STATUS_BAD_SEQLEN);
            else c = (T + kNk - 1) / kNk + ovh;
        }
        // block inclusive scan
        int v = c;
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, v, o);
            if ((threadIdx.x & 31) >= o) v += y;
        }
        if ((threadIdx.x & 31) == 31) warp_sums[threadIdx.x / 32] = v;
        __syncthreads();
        if (threadIdx.x < 32) {
            int w = threadIdx.x < (blockDim.x + 31) / 32 ? warp_sums[threadIdx.x] : 0;
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, w, o);
                if (threadIdx.x >= o) w += y;
            }
            warp_sums[threadIdx.x] = w;
        }
        __syncthreads();
        const int wid = threadIdx.x / 32;
        const int incl = v + (wid > 0 ? warp_sums[wid - 1] : 0) + carry;
        if (b < B) pre[b + 1] = incl;
        __syncthreads();
        if (threadIdx.x == blockDim.x - 1) carry = incl;
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        const int total = pre[B];
        int L = (total + clusters - 1) / clusters;
        if (L < min_units) L = min_units;
        if (L < 1) L = 1;
        plan->L = L;
        plan->ovh = ovh;
        plan->B = B;
        plan->total = total;
    }
}

// ------------------------------------------------------------------ combine

// One warp per (b, i, h) of a sequence cut across clusters: o_lat =
// sum_s 2^(lse_s - lse_max) o_s / sum_s 2^(lse_s - lse_max).  Sequences with
// an invalid length get o_lat = 0.  Sequences done by one cluster are skipped.
__global__ void mla_combine_kernel(const Plan* __restrict__ plan, const float* __restrict__ part_o,
                                   const float* __restrict__ part_lse, int q_len, __nv_bfloat16* __restrict__ o_lat) {
    const int gw = (blockIdx.x * blockDim.x + threadIdx.x) / 32;
    const int lane = threadIdx.x & 31;
    const int B = plan->B;
    if (gw >= B * q_len * kHeads) return;
    const int h = gw % kHeads;
    const int u = gw / kHeads;
    const int b = u / q_len, qi = u % q_len;
    const int* pre = plan_prefix(plan);
    const int L = plan->L, ovh = plan->ovh;
    const int t = plan_tiles(pre, b, ovh);
    __nv_bfloat16* dst = o_lat + ((size_t)u * kHeads + h) * kLat;
    if (t == 0) {
        for (int c = lane * 8; c < kLat; c += 256) *reinterpret_cast<uint4*>(dst + c) = make_uint4(0, 0, 0, 0);
        return;
    }
    const int c_lo = pre[b], c_hi = pre[b + 1];
    const int p0 = c_lo / L, p1 = (c_hi - 1) / L;
    // whole sequence in one cluster?
    int pieces = 0;
    for (int p = p0; p <= p1; ++p) {
        int s = p * L - c_lo - ovh, e = (p + 1) * L - c_lo - ovh;
        s = s < 0 ? 0 : (s > t ? t : s);
        e = e < 0 ? 0 : (e > t ? t : e);
        if (e > s) ++pieces;
    }
    if (pieces <= 1) return;
    float mx = -CUDART_INF_F;
    for (int p = p0; p <= p1; ++p) {
        int s = p * L - c_lo - ovh, e = (p + 1) * L - c_lo - ovh;
        s = s < 0 ? 0 : (s > t ? t : s);
        e = e < 0 ? 0 : (e > t ? t : e);
        if (e > s) mx = fmaxf(mx, part_lse[((size_t)(p + b) * q_len + qi) * kHeads + h]);
    }
    float acc[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) acc[j] = 0.f;
    float wsum = 0.f;
    for (int p = p0; p <= p1; ++p) {
        int s = p * L - c_lo - ovh, e = (p + 1) * L - c_lo - ovh;
        s = s < 0 ? 0 : (s > t ? t : s);
        e = e < 0 ? 0 : (e > t ? t : e);
        if (e <= s) continue;
        const size_t slot = (size_t)(p + b) * q_len + qi;
        const float lse = part_lse[slot * kHeads + h];
        const float w = (lse == -CUDART_INF_F) ? 0.f : exp2f(lse - mx);
        wsum += w;
        const float* src = part_o + (slot * kHeads + h) * kLat;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float4 v = *reinterpret_cast<const float4*>(src + j * 128 + lane * 4);
            acc[4 * j] += w * v.x;
            acc[4 * j + 1] += w * v.y;
            acc[4 * j + 2] += w * v.z;
            acc[4 * j + 3] += w * v.w;
        }
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint2 o;
        o.x = pack_bf16(acc[4 * j] * inv, acc[4 * j + 1] * inv);
        o.y = pack_bf16(acc[4 * j + 2] * inv, acc[4 * j + 3] * inv);
        *reinterpret_cast<uint2*>(dst + j * 128 + lane * 4) = o;
    }
}

}  // namespace sm100
}  // namespace mla
