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
// Work split.  The fp32 accumulator of all 128 heads x 512 latent columns
// would fill the whole 512-column TMEM, leaving no room for S.  A cluster of
// two CTAs therefore splits the 576-wide cache row: CTA "half" 0 takes latent
// columns 0..255 and RoPE columns 0..31, CTA 1 takes 256..511 and 32..63.
// Each computes a partial S over its 288 columns, the pair swaps partial S
// through distributed shared memory (st.async completing on the peer's
// mbarrier), both add the two halves in the same order, run the same
// softmax, and each accumulates its 256 latent columns of O in TMEM.  The
// cache is read from HBM exactly once.  With q_len query tokens the cluster
// holds q_len such pairs that stream the same cache tiles together.
//
// Scheduling (split-KV).  Sequences are cut into 64-key tiles; the clusters
// divide the concatenated tile list into equal contiguous ranges (a fixed
// per-sequence overhead is charged so tiny pieces are avoided).  A sequence
// processed by one cluster writes its normalised o_lat directly (bf16); a
// sequence cut across clusters writes fp32 partials plus a base-2 LSE per
// head, merged by the combine kernel.
//
// Roles per CTA (192 threads): warp 0 TMA producer, warp 1 TMEM owner and
// MMA issuer, warps 2..5 softmax (warp w owns TMEM lanes 32*(w%4)..+31, i.e.
// heads).  Every wait is bounded; on expiry the kernel flags
// MLA_STATUS_TIMEOUT, stops issuing work and tears down normally.
#pragma once

#include <cuda_bf16.h>
#include <math_constants.h>

#include "sm100_ptx.cuh"

namespace mla {
namespace sm100 {

constexpr int kNk = 64;          // keys per tile
constexpr int kHeads = 128;      // M
constexpr int kLat = 512;        // d_c
constexpr int kRope = 64;        // d_r
constexpr int kRow = kLat + kRope;
constexpr int kHalfLat = 256;
constexpr int kHalfRope = 32;

// Shared-memory map (offsets from a 1024-aligned base): a ring of cache
// tiles (each: 4 SW128 chunks of 64 keys x 64 latent columns, then one SW64
// chunk of 64 keys x 32 RoPE columns) and two buffers in which this CTA
// publishes its partial scores for the peer to read.  Q-hat and P live in
// tensor memory.
constexpr int kTileBytes = kNk * 128 * 4 + kNk * 64;       // 36864
constexpr int kStages = 5;
constexpr int kXBytes = kHeads * kNk * 2;                  // 128 x 64 fp16 partial scores
constexpr int kOffTiles = 0;
constexpr int kOffX = kOffTiles + kStages * kTileBytes;    // two publish buffers
constexpr int kOffBars = kOffX + 2 * kXBytes;
constexpr int kAttSmem = kOffBars + 256 + 1024;
// Tensor-memory map (columns of 32 bits, 128 lanes = heads).
constexpr int kTmemCols = 512;
constexpr int kTmemO = 0;      // O: 256 fp32 latent columns of this half
constexpr int kTmemS = 256;    // S: 64 fp32 scores (partial, this half's 288 columns)
constexpr int kTmemP = 320;    // P: 64 bf16 probabilities, two per column
constexpr int kTmemQ = 352;    // Q-hat half: 256 latent + 32 RoPE bf16, two per column (144 columns)
constexpr int kAttThreads = 192;

// Barrier indices (8 bytes each) inside the barrier block.
enum {
    kBarFull0 = 0,
    kBarEmpty0 = kBarFull0 + kStages,
    kBarQFull = kBarEmpty0 + kStages,
    kBarQEmpty,
    kBarSFull,
    kBarSFree,
    kBarPFull,
    kBarPFree,
    kBarOFull,
    kBarOFree,
    kBarXReady0,  // peer has published its partial S in its buffer 0 / 1
    kBarXReady1,
    kBarXRead0,   // peer has finished reading our buffer 0 / 1
    kBarXRead1,
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
    mla_attend_kernel(const __grid_constant__ CUtensorMap mapCacheLat, const __grid_constant__ CUtensorMap mapCacheRope,
                      AttendArgs args) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* base_ptr = smem_raw + (base - raw);
    auto bar = [&](int i) { return base + kOffBars + 8u * i; };
    const uint32_t tmem_slot = bar(kNumBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(base_ptr + kOffBars + 8 * (kNumBars + 1));

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const uint32_t crank = cluster_ctarank();
    const int half = crank & 1;
    const int qi = crank >> 1;
    const uint32_t peer = crank ^ 1u;
    const int cl = (int)cluster_id_x();
    const int q_len = args.q_len;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar(kBarFull0 + s), 1);
            mbar_init(bar(kBarEmpty0 + s), 1);
        }
        mbar_init(bar(kBarQFull), 4);
        mbar_init(bar(kBarQEmpty), 1);
        mbar_init(bar(kBarSFull), 1);
        mbar_init(bar(kBarSFree), 4);
        mbar_init(bar(kBarPFull), 4);
        mbar_init(bar(kBarPFree), 1);
        mbar_init(bar(kBarOFull), 1);
        mbar_init(bar(kBarOFree), 4);
        mbar_init(bar(kBarXReady0), 4);
        mbar_init(bar(kBarXReady1), 4);
        mbar_init(bar(kBarXRead0), 4);
        mbar_init(bar(kBarXRead1), 4);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&mapCacheLat);
        prefetch_tensormap(&mapCacheRope);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    // Peer barriers must be initialised before any remote arrive / st.async.
    cluster_sync();
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
                for (int c = 0; c < 4; ++c)
                    tma_load_3d(dst + c * (kNk * 128), &mapCacheLat, bar(kBarFull0 + st), half * kHalfLat + 64 * c,
                                w.t * kNk, w.seq);
                tma_load_3d(dst + 4 * (kNk * 128), &mapCacheRope, bar(kBarFull0 + st), kLat + half * kHalfRope,
                            w.t * kNk, w.seq);
                MLA_TRACE_POINT(0, n);
            }
        }
    } else if (warp == 1) {
        // ======================================================== MMA issuer (whole warp waits, lane 0 issues)
        constexpr uint32_t idS = idesc_bf16_f32(128, kNk, false, false);
        constexpr uint32_t idO = idesc_bf16_f32(128, kHalfLat, false, true);
        bool ok = true;
        // O(g) += P(g) . C(g); its first K-step overwrites O at the start of a piece.
        auto issue_O = [&](int g, bool first_in_seg, bool last_in_seg) {
            const uint32_t ptile = base + kOffTiles + (g % kStages) * kTileBytes;
            for (int k = 0; k < 4; ++k) {
                const uint64_t bd = smem_desc(ptile + 2048 * k, kNk * 128, 1024, kSw128);
                mma_f16_ts(tmem + kTmemO, tmem + kTmemP + 8 * k, bd, idO, (!first_in_seg || k > 0) ? 1u : 0u);
            }
            mma_commit(bar(kBarPFree));
            mma_commit(bar(kBarEmpty0 + (g % kStages)));
            if (last_in_seg) mma_commit(bar(kBarOFull));
        };
        TileWalk w;
        w.init(args.plan, cl);
        bool prev_first = false, prev_last = false;
        int prev_seg = 0;
        int g = 0;
        for (; w.valid && ok && !*abort_flag; ++g, w.advance()) {
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
                for (int r = r0 + (lane >> 3); r < kNk; r += 4) {
                    for (int c = 0; c < 4; ++c)
                        st_shared_v4(tile + c * (kNk * 128) + r * 128 + (lane & 7) * 16, 0, 0, 0, 0);
                    if ((lane & 7) < 4) st_shared_v4(tile + 4 * (kNk * 128) + r * 64 + (lane & 7) * 16, 0, 0, 0, 0);
                }
                fence_proxy_async_smem();
            }
            __syncwarp();
            // S(g) reuses the S columns: the softmax warps must have read S(g-1).
            if (g > 0 && !mbar_wait(bar(kBarSFree), (g - 1) & 1)) { ok = false; break; }
            tc_fence_after();
            MLA_TRACE_POINT(2, g);
            if (lane == 0) {
                // S = Qhat_half . C_half^T: 4 latent chunks x 4 K-steps, then 2 RoPE K-steps
                for (int c = 0; c < 4; ++c)
                    for (int k = 0; k < 4; ++k) {
                        const uint64_t bd = smem_desc(tile + c * (kNk * 128) + 32 * k, 16, 1024, kSw128);
                        mma_f16_ts(tmem + kTmemS, tmem + kTmemQ + 8 * (4 * c + k), bd, idS, (c | k) ? 1u : 0u);
                    }
                for (int k = 0; k < 2; ++k) {
                    const uint64_t bd = smem_desc(tile + 4 * (kNk * 128) + 32 * k, 16, 512, kSw64);
                    mma_f16_ts(tmem + kTmemS, tmem + kTmemQ + 128 + 8 * k, bd, idS, 1u);
                }
                mma_commit(bar(kBarSFull));
            }
            __syncwarp();
            MLA_TRACE_POINT(3, g);
            if (g > 0) {
                if (!mbar_wait(bar(kBarPFull), (g - 1) & 1)) { ok = false; break; }
                if (prev_first && prev_seg > 0 && !mbar_wait(bar(kBarOFree), (prev_seg - 1) & 1)) { ok = false; break; }
                tc_fence_after();
                MLA_TRACE_POINT(4, g - 1);
                if (lane == 0) issue_O(g - 1, prev_first, prev_last);
                __syncwarp();
                MLA_TRACE_POINT(5, g - 1);
            }
            prev_first = w.first();
            prev_last = w.last();
            prev_seg = w.seg;
        }
        if (ok && !*abort_flag && g > 0) {
            if (!mbar_wait(bar(kBarPFull), (g - 1) & 1)) ok = false;
            else if (prev_first && prev_seg > 0 && !mbar_wait(bar(kBarOFree), (prev_seg - 1) & 1)) ok = false;
            else {
                tc_fence_after();
                if (lane == 0) issue_O(g - 1, prev_first, prev_last);
                __syncwarp();
            }
        }
        if (!ok) *abort_flag = 1;
    } else {
        // ======================================================== softmax warps 2..5 (row r = head r)
        // Software pipeline: iteration g publishes the partial scores of tile
        // g+1 before it runs the softmax of tile g, so the exchange with the
        // peer overlaps a whole iteration.  Each CTA writes its fp16 partial
        // scores into its own shared memory and the peer pulls them with
        // ld.shared::cluster; one remote arrive per warp signals "published"
        // and one signals "read".
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        const uint32_t x_local = base + kOffX;
        const uint32_t x_peer = mapa(x_local, peer);
        const uint32_t xready_peer0 = mapa(bar(kBarXReady0), peer);
        const uint32_t xread_peer0 = mapa(bar(kBarXRead0), peer);
        const float sl2 = args.scale_log2;
        bool ok = true;

        // this half of Q-hat row r -> TMEM columns kTmemQ.. (144 columns)
        auto load_q = [&](int seq) {
            const int u = seq * q_len + qi;
            const uint4* src = reinterpret_cast<const uint4*>(args.q_hat + ((size_t)u * kHeads + r) * kRow);
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t v[32];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint4 x = __ldg(src + half * 32 + c * 8 + j);
                    v[4 * j] = x.x; v[4 * j + 1] = x.y; v[4 * j + 2] = x.z; v[4 * j + 3] = x.w;
                }
                tmem_st32(tmem + lane_addr + kTmemQ + 32 * c, v);
            }
            uint32_t v[16];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint4 x = __ldg(src + 64 + half * 4 + j);
                v[4 * j] = x.x; v[4 * j + 1] = x.y; v[4 * j + 2] = x.z; v[4 * j + 3] = x.w;
            }
            tmem_st16(tmem + lane_addr + kTmemQ + 128, v);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kBarQFull));
        };
        // partial S(g) out of TMEM, scaled to log2 units, published as fp16 in
        // our buffer g & 1; own copy kept (rounded the same way) in `mine`.
        auto fetch_send = [&](int g, uint32_t (&mine)[32]) -> bool {
            if (!mbar_wait(bar(kBarSFull), g & 1)) return false;
            tc_fence_after();
            MLA_TRACE_POINT(7, g);
            uint32_t v[32], v2[32];
            tmem_ld32(tmem + lane_addr + kTmemS, v);
            tmem_ld32(tmem + lane_addr + kTmemS + 32, v2);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kBarSFree));
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                mine[j] = pack_f16(__uint_as_float(v[2 * j]) * sl2, __uint_as_float(v[2 * j + 1]) * sl2);
                mine[16 + j] = pack_f16(__uint_as_float(v2[2 * j]) * sl2, __uint_as_float(v2[2 * j + 1]) * sl2);
            }
            const int b = g & 1;
            // the peer must have finished reading what we published in this buffer two tiles ago
            if (g >= 2 && !mbar_wait_cluster(bar(kBarXRead0 + b), ((g - 2) >> 1) & 1)) return false;
            MLA_TRACE_POINT(8, g);
            const uint32_t dst = x_local + b * kXBytes + r * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c)
                st_shared_v4(dst + ((c ^ (r & 7)) << 4), mine[4 * c], mine[4 * c + 1], mine[4 * c + 2], mine[4 * c + 3]);
            fence_acq_rel_cluster();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(xready_peer0 + 8 * b);
            MLA_TRACE_POINT(9, g);
            return true;
        };

        TileWalk cur, nxt;
        cur.init(args.plan, cl);
        nxt = cur;
        uint32_t mine_cur[32], mine_nxt[32];
        if (cur.valid) {
            load_q(cur.seq);
            ok = fetch_send(0, mine_cur);
            nxt.advance();
        }
        float m_used = -CUDART_INF_F, l_sum = 0.f;
        int g = 0;
        for (; cur.valid && ok && !*abort_flag; ++g) {
            if (nxt.valid) {
                if (nxt.seg != cur.seg) load_q(nxt.seq);  // S(g) was read: Q-hat columns are free
                if (!fetch_send(g + 1, mine_nxt)) { ok = false; break; }
            }
            // ---- pull the peer's partial S(g) and add it (half 0's part first)
            const int b = g & 1;
            if (!mbar_wait_cluster(bar(kBarXReady0 + b), (g >> 1) & 1)) { ok = false; break; }
            MLA_TRACE_POINT(10, g);
            float s[kNk];
            const uint32_t src = x_peer + b * kXBytes + r * 128;
            uint32_t xs[32];
#pragma unroll
            for (int c = 0; c < 8; ++c)
                ld_cluster_v4u(src + ((c ^ (r & 7)) << 4), xs[4 * c], xs[4 * c + 1], xs[4 * c + 2], xs[4 * c + 3]);
#pragma unroll
            for (int q = 0; q < 32; ++q) {
                const float2 o = unpack_f16(xs[q]);
                const float2 m = unpack_f16(mine_cur[q]);
                s[2 * q] = half == 0 ? m.x + o.x : o.x + m.x;
                s[2 * q + 1] = half == 0 ? m.y + o.y : o.y + m.y;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(xread_peer0 + 8 * b);
            // ---- online softmax in base 2 with lazy rescaling of O
            const int T_b = args.seqlens[cur.seq];
            const int n_keys = T_b - q_len + 1 + qi;  // query qi attends to keys 0..n_keys-1
            const int key0 = cur.t * kNk;
            if (key0 + kNk > n_keys) {
#pragma unroll
                for (int j = 0; j < kNk; ++j)
                    if (key0 + j >= n_keys) s[j] = -CUDART_INF_F;
            }
            float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
            for (int j = 4; j < kNk; j += 4) {
                mx0 = fmaxf(mx0, s[j]); mx1 = fmaxf(mx1, s[j + 1]);
                mx2 = fmaxf(mx2, s[j + 2]); mx3 = fmaxf(mx3, s[j + 3]);
            }
            const float mx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
            const bool first = cur.first();
            const bool grow = mx > m_used + 8.0f;  // rescale only when the max grows by > 2^8
            const float mb_new = grow ? mx : m_used;
            const float mb = (mb_new == -CUDART_INF_F) ? 0.f : mb_new;
            uint32_t pk[32];
            float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float p0 = ex2(s[2 * j] - mb), p1 = ex2(s[2 * j + 1] - mb);
                rs0 += p0;
                rs1 += p1;
                pk[j] = pack_bf16(p0, p1);
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
            l_sum += rs0 + rs1;
            tmem_st32(tmem + lane_addr + kTmemP, pk);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kBarPFull));
            MLA_TRACE_POINT(13, g);
            // ---- epilogue at the end of a piece
            if (cur.last()) {
                if (!mbar_wait(bar(kBarOFull), cur.seg & 1)) { ok = false; break; }
                tc_fence_after();
                const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
                const int u = cur.seq * q_len + qi;
                if (cur.whole) {
                    __nv_bfloat16* dst = args.o_lat + ((size_t)u * kHeads + r) * kLat + half * kHalfLat;
#pragma unroll 1
                    for (int c0 = 0; c0 < kHalfLat; c0 += 32) {
                        uint32_t v[32];
                        tmem_ld32(tmem + lane_addr + kTmemO + c0, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 32; j += 8) {
                            uint4 w;
                            w.x = pack_bf16(__uint_as_float(v[j]) * inv, __uint_as_float(v[j + 1]) * inv);
                            w.y = pack_bf16(__uint_as_float(v[j + 2]) * inv, __uint_as_float(v[j + 3]) * inv);
                            w.z = pack_bf16(__uint_as_float(v[j + 4]) * inv, __uint_as_float(v[j + 5]) * inv);
                            w.w = pack_bf16(__uint_as_float(v[j + 6]) * inv, __uint_as_float(v[j + 7]) * inv);
                            *reinterpret_cast<uint4*>(dst + c0 + j) = w;
                        }
                    }
                } else {
                    const int slot = cl + cur.seq;
                    float* dst = args.part_o + (((size_t)slot * q_len + qi) * kHeads + r) * kLat + half * kHalfLat;
#pragma unroll 1
                    for (int c0 = 0; c0 < kHalfLat; c0 += 32) {
                        uint32_t v[32];
                        tmem_ld32(tmem + lane_addr + kTmemO + c0, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 32; j += 4) {
                            float4 w = make_float4(__uint_as_float(v[j]) * inv, __uint_as_float(v[j + 1]) * inv,
                                                   __uint_as_float(v[j + 2]) * inv, __uint_as_float(v[j + 3]) * inv);
                            *reinterpret_cast<float4*>(dst + c0 + j) = w;
                        }
                    }
                    if (half == 0)
                        args.part_lse[((size_t)slot * q_len + qi) * kHeads + r] =
                            l_sum > 0.f ? m_used + __log2f(l_sum) : -CUDART_INF_F;
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kBarOFree));
                m_used = -CUDART_INF_F;
                l_sum = 0.f;
            }
            // advance the pipeline
#pragma unroll
            for (int j = 0; j < 32; ++j) mine_cur[j] = mine_nxt[j];
            cur = nxt;
            if (nxt.valid) nxt.advance();
        }
        if (!ok) *abort_flag = 1;
    }

    if (*abort_flag && threadIdx.x == 0) atomicOr(args.status, MLA_STATUS_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, kTmemCols);
    // The peer may still read our barriers / write our X buffers until it is done.
    cluster_sync();
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
