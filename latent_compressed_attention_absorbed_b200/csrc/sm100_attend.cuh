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
// Work split.  The fp32 accumulator of 128 heads x 512 latent columns would
// fill all 512 TMEM columns of an SM, and an M = 64 MMA runs at half the
// tensor rate, so a CTA keeps all 128 heads (M = 128) and a cluster of two
// CTAs splits the 576-wide cache row: CTA r loads and multiplies latent
// columns 256r..256r+255 and RoPE columns 32r..32r+31 of every tile (the
// cache crosses HBM and L2 once).  Each CTA computes a partial S over its
// 288 columns, scales it to log2 units and rounds it to fp16; the pair swaps
// the rounded partials through distributed shared memory (one bulk copy per
// warp), both add the two halves (fp32 addition is commutative, so both CTAs
// see the same S), run the same online softmax, and each accumulates its
// 256 latent columns of O in TMEM.
//
// Scheduling (split-KV).  Sequences are cut into 64-key tiles.  The clusters
// form groups of q_len (cluster c: group c / q_len, query token c % q_len);
// the groups divide the concatenated tile list of all sequences into equal
// contiguous ranges (a fixed per-sequence overhead is charged so tiny pieces
// are avoided), and the q_len clusters of a group stream the same tiles at
// the same time, so L2 serves the repeats.  A sequence processed by one
// group writes its normalised o_lat directly (bf16); a sequence cut across
// groups writes fp32 partials plus a base-2 LSE per head and token, merged by
// the combine kernel.
//
// Roles per CTA (512 threads; warps 12-15 are the second softmax warp of each
// quarter, warp 11 is idle):
//   warp 0     TMA producer (stage ring, L2 prefetch of the tiles ahead);
//   warp 1     TMEM owner and issuer of the score MMAs (S);
//   warp 10    issuer of the P.V MMAs (O), as soon as P is published;
//   warps 2-5, softmax, two warps per TMEM lane quarter (32 keys each): add
//   12-15      the two partial scores, online softmax, P into TMEM, rescale /
//              normalise O, write o_lat or split partials;
//   warps 6-9  exchange: read partial S out of TMEM, publish it (local copy
//              for the softmax warps, bulk copy to the peer), load Q-hat.
// Warp w reaches TMEM lanes 32*(w%4)..+31; lane l of warp w owns head
// 32*(w%4)+l, a whole score row.  Every wait is bounded; on expiry the
// kernel flags MLA_STATUS_TIMEOUT, stops issuing work and tears down
// normally (the two softmax warps of a quarter, which meet on a named
// barrier, decide together whether to stop, so neither is left waiting).
#pragma once

#include <cuda_bf16.h>
#include <math_constants.h>

#include <climits>

#include "mla_rope.cuh"
#include "sm100_ptx.cuh"

namespace mla {
namespace sm100 {

constexpr int kNk = 64;      // keys per tile
constexpr int kHeads = 128;  // heads of a token (M of every MMA)
constexpr int kLat = 512;    // d_c
constexpr int kRope = 64;    // d_r
constexpr int kRow = kLat + kRope;
constexpr int kHalfLat = 256;
constexpr int kHalfRope = 32;

// Shared-memory map (offsets from a 1024-aligned base).
//   stages: ring of this CTA's half tiles: 4 SW128 chunks of 64 keys x 64
//           latent columns, then 64 keys x 32 RoPE columns (SW64);
//   Own:    two buffers of this CTA's partial scores, 128 x 64 fp16 (rows of
//           128 bytes, 16-byte chunks swizzled by row), read by the local
//           softmax warps and bulk-copied to the peer's X buffer;
//   X:      two buffers receiving the peer's partial scores (same layout);
//   QR:     this CTA's RoPE half of Q-hat, 128 heads x 32 bf16 (SW64).
constexpr int kChunk = kNk * 128;                     // 8192
constexpr int kRopeChunk = kNk * 64;                  // 4096
constexpr int kStageBytes = 4 * kChunk + kRopeChunk;  // 36864
constexpr int kStages = 4;
#ifndef MLA_PREFETCH_TILES
#define MLA_PREFETCH_TILES 6
#endif
constexpr int kPrefetch = MLA_PREFETCH_TILES;  // tiles prefetched into L2 ahead of the stage loads
constexpr int kXBytes = kHeads * 128;                 // 16384
constexpr int kOffStages = 0;
constexpr int kOffOwn = kOffStages + kStages * kStageBytes;
constexpr int kOffX = kOffOwn + 2 * kXBytes;
constexpr int kQRBytes = kHeads * 64;                  // 8192
constexpr int kOffQR = kOffX + 2 * kXBytes;
constexpr int kOffRed = kOffQR + kQRBytes;            // softmax pair exchange: [2][2][128] fp32
constexpr int kOffFlags = kOffRed + 2 * 2 * kHeads * 4;  // softmax pair status: [2][4 quarters][2] int
constexpr int kOffBars = kOffFlags + 2 * 4 * 2 * 4;
constexpr int kAttSmem = kOffBars + 256 + 1024;
static_assert(kAttSmem <= 232448, "attention kernel shared memory exceeds 227 KB");

// Tensor-memory map: 512 columns of 32 bits, lane = head.
constexpr int kTmemCols = 512;
constexpr int kTmemO = 0;     // O: 256 fp32 latent columns of this CTA's half
constexpr int kTmemS = 256;   // S: 64 fp32 partial scores
constexpr int kTmemP = 320;   // P: two buffers of 64 bf16 probabilities, two per column
constexpr int kTmemQ = 384;   // Q-hat latent half: 256 bf16, two per column (128 columns)
constexpr int kAttThreads = 512;

// Barrier indices (8 bytes each) inside the barrier block.
enum {
    kBarFull0 = 0,
    kBarEmpty0 = kBarFull0 + kStages,
    kBarQFull = kBarEmpty0 + kStages,  // Q-hat of the next piece loaded (4 exchange warps + RoPE-half TMA)
    kBarSFull,                         // S(g) complete (MMA commit)
    kBarSFree,                         // S(g) read out of TMEM (4 exchange warps)
    kBarPFull0,                        // P(g) in TMEM buffer g%2 (4 softmax warps)
    kBarPFree0 = kBarPFull0 + 2,       // O(g) complete: P buffer g%2 (and O) may be touched (MMA commit)
    kBarOwnFull0 = kBarPFree0 + 2,     // own partial g in Own[g%2] (4 exchange warps)
    kBarOwnFree0 = kBarOwnFull0 + 2,   // Own[g%2] read by the softmax warps (4)
    kBarXFull0 = kBarOwnFree0 + 2,     // peer's partial g landed in X[g%2] (tx)
    kBarXFree0 = kBarXFull0 + 2,       // the peer has read what we sent into its X[g%2] (4, remote)
    kBarOFull = kBarXFree0 + 2,        // last O of a piece complete (MMA commit)
    kBarOFree,                         // O read by the epilogue (8 softmax warps)
    kNumBars
};
static_assert(8 * (kNumBars + 2) <= 256, "barrier block too small");

// Optional timing trace (compile with -DMLA_TRACE): global-timer stamps (ns)
// of both CTAs of one cluster at fixed points of every tile, read back by
// mla_trace_read.  Events: 0 tile loads issued, 1 S issued, 2 O issued,
// 3 S read by the exchange warps, 4 own partial published, 5 both partials
// available to the softmax warps, 6 P published, 7 piece epilogue done,
// 8 row max, 9 P computed, 10 tile data seen by the MMA warp, 11..13 P
// published by warps 3, 4, 5.
#ifdef MLA_TRACE
#ifndef MLA_TRACE_CLUSTER
#define MLA_TRACE_CLUSTER 0
#endif
constexpr int kTraceTiles = 4096;
constexpr int kTraceProlog = kTraceTiles - 1;  // row of kernel-level stamps
__device__ unsigned long long g_mla_trace[2][kTraceTiles][16];
#define MLA_TRACE_POINT(ev, n)                                                                            \
    do {                                                                                                  \
        if (cl == MLA_TRACE_CLUSTER && (n) < kTraceTiles) g_mla_trace[r][(n)][(ev)] = global_timer_ns(); \
    } while (0)
// Per-CTA summary of every cluster: [cluster][rank][24] = entry, after the
// grid dependency wait, first S issued, last O issued, last epilogue done,
// exit, tiles, pieces, SM id, then clock cycles spent in the barrier waits
// listed at kTw* (one representative thread per role).
constexpr int kTraceAllClusters = 256;
__device__ unsigned long long g_mla_trace_all[kTraceAllClusters][2][24];
enum {
    kTwFull,      // S issuer: tile data
    kTwSFree,     // S issuer: previous S read out of TMEM
    kTwQFull,     // S issuer: Q-hat of a piece
    kTwSFull,     // exchange: S complete
    kTwOwnFree,   // exchange: buffers of tile h-2 released (own and peer)
    kTwXFull,     // softmax: own and peer partials
    kTwPFree,     // softmax: P buffer released by O(g-2) (and O ready for a rescale)
    kTwPFull,     // O issuer: P published
    kTwOFree,     // O issuer: previous piece's O read
    kTwEmpty,     // producer: stage released
    kTwN
};
constexpr int kTwBase = 9;
#ifdef MLA_TRACE_WAITS
#define MLA_TW(slot, call) mla_tw_(tw_acc[(slot)], [&]() { return (bool)(call); })
#else
#define MLA_TW(slot, call) (call)
#endif
template <class F>
__device__ __forceinline__ bool mla_tw_(unsigned long long& acc, F f) {
    const long long t0 = clock64();
    const bool ok = f();
    acc += (unsigned long long)(clock64() - t0);
    return ok;
}
#define MLA_TRACE_ALL(ev, value)                                         \
    do {                                                                 \
        if (cl < kTraceAllClusters) g_mla_trace_all[cl][r][(ev)] = (value); \
    } while (0)
// Kernel timeline of the decode step: [kernel][first entry, first return
// from the grid dependency wait, last exit], stamped by thread 0 of each CTA.
enum { kKtAppend, kKtAbsorb, kKtAttend, kKtCombine, kKtProject, kKtN };
__device__ unsigned long long g_mla_ktrace[kKtN][3];
#define MLA_KT(k, ev)                                                                       \
    do {                                                                                    \
        if (threadIdx.x == 0) {                                                             \
            if ((ev) < 2) atomicMin(&::mla::sm100::g_mla_ktrace[k][ev], global_timer_ns()); \
            else atomicMax(&::mla::sm100::g_mla_ktrace[k][ev], global_timer_ns());          \
        }                                                                                   \
    } while (0)
#else
#define MLA_KT(k, ev) \
    do {              \
    } while (0)
#define MLA_TRACE_ALL(ev, value) \
    do {                         \
    } while (0)
#define MLA_TW(slot, call) (call)
#define MLA_TRACE_POINT(ev, n) \
    do {                       \
    } while (0)
#endif
// Kernel-level stamps (row kTraceProlog): 0 entry, 1 after set-up, 2 after the
// grid dependency wait, 3 first Q-hat loaded, 4 epilogue start, 5 epilogue
// end, 6 teardown start, 7 exit.

// Scheduling plan written by the plan warp into the workspace.
struct Plan {
    int L;        // cost units per group
    int ovh;      // cost charged per sequence
    int B;        // sequences
    int total;    // sum of costs
    int n_split;  // sequences cut across groups (listed after the prefix sums)
    int q_len;
    int groups;   // groups of q_len clusters
    int pad;
    // followed by int group_first[kPlanMaxGroups] (the sequence holding cost
    // unit g L, or B past the end), int cost_prefix[B + 1], int split_seq[B]
};
// The per-group table sits at a fixed offset, so that a cluster finds its
// first piece without a search over the prefix sums: the header, the table
// entry and then two prefix sums are two dependent reads from global memory.
constexpr int kPlanMaxGroups = 1024;  // the cluster count is capped at 1024

__device__ __forceinline__ const int* plan_group_first(const Plan* p) { return reinterpret_cast<const int*>(p + 1); }
__device__ __forceinline__ const int* plan_prefix(const Plan* p) { return plan_group_first(p) + kPlanMaxGroups; }
__device__ __forceinline__ const int* plan_splits(const Plan* p) { return plan_prefix(p) + p->B + 1; }

// Tiles of sequence b (0 if its length was invalid).
__device__ __forceinline__ int plan_tiles(const int* pre, int b, int ovh) {
    const int c = pre[b + 1] - pre[b];
    return c > 0 ? c - ovh : 0;
}

// Segment iterator: the (sequence, tile range) pieces of group `grp`.
struct SegIter {
    const int* pre;
    int B, L, ovh, lo, hi, b;
    __device__ void init(const Plan* plan, int grp) {
        pre = plan_prefix(plan);
        B = plan->B;
        L = plan->L;
        ovh = plan->ovh;
        lo = grp * L;
        hi = lo + L;
        b = plan_group_first(plan)[grp];  // the sequence whose cost range holds lo
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

// Flat walk over the tiles of a group's pieces, with the piece's bounds.
struct TileWalk {
    SegIter it;
    int seq, k0, k1, t, seg;
    bool whole, valid;
    __device__ void init(const Plan* plan, int grp) {
        it.init(plan, grp);
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
    float scale_log2;             // softmax_scale * log2(e)
    const __nv_bfloat16* q_hat;   // [B][q_len][128][576]
    __nv_bfloat16* o_lat;         // [B][q_len][128][512]
    int o_lat_v8;                 // o_lat is 32-byte aligned: 32-byte stores
    const uint8_t* prefetch;      // optional: range prefetched into L2 while the kernel runs
    size_t prefetch_bytes;        // (the next step's weights when this step's own traffic is small)
    float* part_o;                // [slots][64 column octets][128 heads][8]
    float* part_lse;              // [slots][128]
    int* status;
};

// Byte offset of 16-byte chunk c of row r in a buffer of 128-byte rows whose
// chunks are permuted by row (c ^ (r % 8)), the SW128 pattern: the 8 rows a
// quarter-warp touches at once land in 8 different bank groups.
__device__ __forceinline__ uint32_t sw128(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

// mapLat: cache [B][T_max][576] bf16, box 64 columns x 64 keys, SW128.
// mapRope: same tensor, box 32 columns x 64 keys, SW64.
// mapPf: the cache again, box 256 columns x 64 keys, no swizzle (L2 prefetch only).
// mapQR: q_hat [U][128][576] bf16, box 32 columns x 128 heads, SW64.
__global__ void __launch_bounds__(kAttThreads, 1)
    mla_attend_kernel(const __grid_constant__ CUtensorMap mapLat, const __grid_constant__ CUtensorMap mapRope,
                      const __grid_constant__ CUtensorMap mapPf, const __grid_constant__ CUtensorMap mapQR,
                      AttendArgs args) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* base_ptr = smem_raw + (base - raw);
    auto bar = [&](int i) { return base + kOffBars + 8u * i; };
    const uint32_t tmem_slot = bar(kNumBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(base_ptr + kOffBars + 8 * (kNumBars + 1));

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const uint32_t r = cluster_ctarank() & 1;  // latent half of this CTA
    const uint32_t peer = r ^ 1;
    const int cl = (int)cluster_id_x();
    const int q_len = args.q_len;
    const int grp = cl / q_len, qi = cl % q_len;

    if (threadIdx.x == 0) MLA_TRACE_POINT(0, kTraceProlog);
    if (threadIdx.x == 0) MLA_TRACE_ALL(0, global_timer_ns());
    MLA_KT(kKtAttend, 0);
#ifdef MLA_TRACE_WAITS
    unsigned long long tw_acc[kTwN];
#pragma unroll
    for (int i = 0; i < kTwN; ++i) tw_acc[i] = 0;
#endif
#ifdef MLA_TRACE
    if (threadIdx.x == 0) {
        unsigned smid;
        asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
        MLA_TRACE_ALL(8, smid);
    }
#endif
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar(kBarFull0 + s), 1);
            mbar_init(bar(kBarEmpty0 + s), 1);
        }
        mbar_init(bar(kBarQFull), 5);
        mbar_init(bar(kBarSFull), 1);
        mbar_init(bar(kBarSFree), 4);
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(kBarPFull0 + s), 8);
            mbar_init(bar(kBarPFree0 + s), 1);
            mbar_init(bar(kBarOwnFull0 + s), 4);
            mbar_init(bar(kBarOwnFree0 + s), 8);
            mbar_init(bar(kBarXFull0 + s), 1);
            mbar_init(bar(kBarXFree0 + s), 8);
        }
        mbar_init(bar(kBarOFull), 1);
        mbar_init(bar(kBarOFree), 8);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&mapLat);
        prefetch_tensormap(&mapRope);
        prefetch_tensormap(&mapPf);
        prefetch_tensormap(&mapQR);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    // The peer's barriers must be initialised before any remote access.
    cluster_sync();
    tc_fence_after();
    if (threadIdx.x == 0) MLA_TRACE_POINT(1, kTraceProlog);
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(base_ptr + kOffBars + 8 * kNumBars);
    // The set-up above overlaps the previous kernel; the plan, Q-hat and the
    // cache are read only once it has completed.
    pdl_wait();
    if (threadIdx.x == 0) pdl_trigger();
    if (threadIdx.x == 0) MLA_TRACE_POINT(2, kTraceProlog);
    if (threadIdx.x == 0) MLA_TRACE_ALL(1, global_timer_ns());
    MLA_KT(kKtAttend, 1);
    const bool active = grp < args.plan->groups;
    // Warp 0, lanes 1..31: spread the optional L2 prefetch over the grid, 16 KB a request.
    if (warp == 0 && lane > 0 && args.prefetch) {
        const size_t per_cta = ((args.prefetch_bytes / gridDim.x) + 16383) & ~size_t(16383);
        const size_t lo = per_cta * blockIdx.x;
        for (size_t off = lo + 16384 * (size_t)(lane - 1); off < lo + per_cta && off < args.prefetch_bytes;
             off += 16384 * 31) {
            const size_t n = args.prefetch_bytes - off < 16384 ? args.prefetch_bytes - off : 16384;
            prefetch_l2_bulk(args.prefetch + off, (uint32_t)(n & ~size_t(15)));
        }
    }

    const int quarter = warp & 3;
    const int m = quarter * 32 + lane;                          // head / TMEM lane (warps 2..9)
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;  // the warp's TMEM subpartition

    if (!active) {
        // idle cluster (the cluster count is not a multiple of q_len)
    } else if (warp == 0) {
        // ======================================================== TMA producer (runs up to kStages tiles ahead)
        // Tiles kPrefetch ahead of the loads are prefetched into L2, so that a
        // stage, once freed, refills at L2 rather than HBM latency.  (Issuing the
        // first loads ahead of the first prefetches measured slower: the early
        // burst of prefetches keeps HBM busy while the pipeline fills.)
        if (lane == 0) {
            TileWalk w, wp;
            w.init(args.plan, grp);
            wp = w;
            for (int i = 0; i < kPrefetch && wp.valid; ++i) {
                tma_prefetch_3d(&mapPf, kHalfLat * r, wp.t * kNk, wp.seq);
                tma_prefetch_3d(&mapRope, kLat + kHalfRope * r, wp.t * kNk, wp.seq);
                wp.advance();
            }
            for (int n = 0; w.valid && !*abort_flag; ++n, w.advance()) {
                if (kPrefetch > 0 && wp.valid) {
                    // A later piece's Q-hat (147 KB, contiguous) goes into L2 as the
                    // look-ahead enters it, ahead of its reload: each CTA of the
                    // pair prefetches one half, 8 KB a request.
                    if (wp.first() && wp.seg > 0) {
                        constexpr uint32_t kQBytes = kHeads * kRow * 2, kPiece = 8192;
                        const uint8_t* q = reinterpret_cast<const uint8_t*>(args.q_hat) +
                                           (size_t)(wp.seq * q_len + qi) * kQBytes;
                        for (uint32_t off = r * (kQBytes / 2); off < (r + 1) * (kQBytes / 2); off += kPiece)
                            prefetch_l2_bulk(q + off, kPiece);
                    }
                    tma_prefetch_3d(&mapPf, kHalfLat * r, wp.t * kNk, wp.seq);
                    tma_prefetch_3d(&mapRope, kLat + kHalfRope * r, wp.t * kNk, wp.seq);
                    wp.advance();
                }
                const int st = n % kStages;
                if (n >= kStages && !MLA_TW(kTwEmpty, mbar_wait(bar(kBarEmpty0 + st), ((n / kStages) - 1) & 1))) {
                    *abort_flag = 1;
                    break;
                }
                const uint32_t dst = base + kOffStages + st * kStageBytes;
                mbar_arrive_expect_tx(bar(kBarFull0 + st), kStageBytes);
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    tma_load_3d(dst + c * kChunk, &mapLat, bar(kBarFull0 + st), kHalfLat * r + 64 * c, w.t * kNk, w.seq);
                tma_load_3d(dst + 4 * kChunk, &mapRope, bar(kBarFull0 + st), kLat + kHalfRope * r, w.t * kNk, w.seq);
                MLA_TRACE_POINT(0, n);
            }
        }
    } else if (warp == 1) {
        // ======================================================== S issuer (whole warp waits, lane 0 issues)
        constexpr uint32_t idS = idesc_bf16_f32(kHeads, kNk, false, false);
        const uint32_t stages = base + kOffStages;
        // Descriptor templates: the start-address field (bits 0..13, address >> 4)
        // is advanced by adding byte offsets >> 4.
        const uint64_t dLatK = smem_desc(stages, 16, 1024, kSw128);       // cache latent, K-major (S)
        const uint64_t dRopeK = smem_desc(stages, 16, 512, kSw64);        // cache RoPE, K-major (S)
        const uint64_t dQR = smem_desc(base + kOffQR, 16, 512, kSw64);    // Q-hat RoPE half (S, A operand)
        // S(g) = Q-hat half . cache half^T over this CTA's 288 columns, in tile
        // order: each S waits for its piece's Q-hat, its tile and S(g-1) to be
        // read out of TMEM.  (The O MMAs are issued by warp 10: issuing blocks
        // at the tensor pipe's pace, and a ready O must not wait behind an S.)
        TileWalk ws;
        ws.init(args.plan, grp);
        int T_s = ws.valid ? args.seqlens[ws.seq] : 0;  // length of the sequence of tile g
        bool ok = true;
        for (int g = 0; ws.valid && ok && !*abort_flag; ++g) {
            if (ws.first() && !MLA_TW(kTwQFull, mbar_wait(bar(kBarQFull), ws.seg & 1))) { ok = false; break; }
            const uint32_t tile_off = kOffStages + (g % kStages) * kStageBytes;
            if (!MLA_TW(kTwFull, mbar_wait(bar(kBarFull0 + g % kStages), (g / kStages) & 1))) { ok = false; break; }
#ifdef MLA_TRACE
            if (lane == 0) MLA_TRACE_POINT(10, g);
#endif
            if (g > 0 && !MLA_TW(kTwSFree, mbar_wait(bar(kBarSFree), (g - 1) & 1))) { ok = false; break; }
            const int valid = T_s - ws.t * kNk;
            if (valid < kNk) {
                // Rows at or beyond T_b hold no cached token: zero the latent
                // part so that masked (p = 0) rows cannot inject NaN/Inf into P.C.
                const int r0 = valid < 0 ? 0 : valid;
                for (int row = r0 + (lane >> 3); row < kNk; row += 4)
                    for (int c = 0; c < 4; ++c)
                        st_shared_v4(base + tile_off + c * kChunk + row * 128 + (lane & 7) * 16, 0, 0, 0, 0);
                fence_proxy_async_smem();
            }
            __syncwarp();
            tc_fence_after();
            if (lane == 0) {
                MLA_TRACE_POINT(14, g);
#ifdef MLA_TRACE_CYCLES
                const long long c_s0 = clock64();
#endif
                const uint32_t dS = tmem + kTmemS;
                const uint64_t dL = dLatK + (tile_off >> 4);
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    mma_f16_ts(dS, tmem + kTmemQ + 8 * k, dL + (((k >> 2) * kChunk + 32 * (k & 3)) >> 4), idS,
                               k ? 1u : 0u);
#pragma unroll
                for (int j = 0; j < 2; ++j)
                    mma_f16_ss(dS, dQR + ((32 * j) >> 4), dRopeK + ((tile_off + 4 * kChunk + 32 * j) >> 4), idS, 1u);
                mma_commit(bar(kBarSFull));
                MLA_TRACE_POINT(1, g);
                if (g == 0) MLA_TRACE_ALL(2, global_timer_ns());
#ifdef MLA_TRACE_CYCLES
                if (cl == MLA_TRACE_CLUSTER && g < kTraceTiles) g_mla_trace[r][g][11] = (unsigned long long)(clock64() - c_s0);
#endif
            }
            __syncwarp();
            const int seq_before = ws.seq;
            ws.advance();
            if (ws.valid && ws.seq != seq_before) T_s = args.seqlens[ws.seq];
        }
        if (!ok) *abort_flag = 1;
    } else if (warp == 10) {
        // ======================================================== O issuer (whole warp waits, lane 0 issues)
        // O += P(g) . cache latent half(g); the first tile of a piece overwrites
        // O (after the previous piece's epilogue has read it).
        constexpr uint32_t idO = idesc_bf16_f32(kHeads, kHalfLat, false, true);
        const uint64_t dLatMN = smem_desc(base + kOffStages, kChunk, 1024, kSw128);  // cache latent, MN-major
        TileWalk wo;
        wo.init(args.plan, grp);
        bool ok = true;
        for (int g = 0; wo.valid && ok && !*abort_flag; ++g, wo.advance()) {
            if (!MLA_TW(kTwPFull, mbar_wait(bar(kBarPFull0 + (g & 1)), (g >> 1) & 1))) { ok = false; break; }
            if (wo.first() && wo.seg > 0 && !MLA_TW(kTwOFree, mbar_wait(bar(kBarOFree), (wo.seg - 1) & 1))) { ok = false; break; }
            tc_fence_after();
            if (lane == 0) {
                MLA_TRACE_POINT(15, g);
                const bool first = wo.first();
                const int st = g % kStages;
                const uint64_t dB = dLatMN + ((kOffStages + st * kStageBytes) >> 4);
                const uint32_t pA = tmem + kTmemP + 32 * (g & 1);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_f16_ts(tmem + kTmemO, pA + 8 * k, dB + ((2048 * k) >> 4), idO, (!first || k > 0) ? 1u : 0u);
                mma_commit(bar(kBarPFree0 + (g & 1)));
                mma_commit(bar(kBarEmpty0 + st));
                if (wo.last()) mma_commit(bar(kBarOFull));
                MLA_TRACE_POINT(2, g);
                MLA_TRACE_ALL(3, global_timer_ns());
                MLA_TRACE_ALL(6, (unsigned long long)(g + 1));
                MLA_TRACE_ALL(7, (unsigned long long)(wo.seg + 1));
            }
            __syncwarp();
        }
        if (!ok) *abort_flag = 1;
    } else if (warp == 11) {
        // spare warp (keeps the softmax halves on the same SMSPs as their quarters)
    } else if (warp >= 6 && warp <= 9) {
        // ======================================================== exchange warps 6..9
        const float sl2 = args.scale_log2;
        const uint32_t x_peer = mapa(base + kOffX, peer);
        const uint32_t xfull_peer = mapa(bar(kBarXFull0), peer);
        bool ok = true;
        // Q-hat of unit u, this CTA's half: row m's 256 latent values -> TMEM
        // (this thread), the 128 x 32 RoPE block -> shared memory by TMA
        // (issued by thread 192).
        auto load_q = [&](int u) {
            if (threadIdx.x == 192) {
                mbar_arrive_expect_tx(bar(kBarQFull), kQRBytes);
                tma_load_3d(base + kOffQR, &mapQR, bar(kBarQFull), kLat + kHalfRope * r, 0, u);
            }
            const uint4* src = reinterpret_cast<const uint4*>(args.q_hat + ((size_t)u * kHeads + m) * kRow) + 32 * r;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint4 x[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) x[j] = __ldg(src + 16 * half + j);
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint32_t v[32];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        v[4 * j] = x[8 * c + j].x; v[4 * j + 1] = x[8 * c + j].y;
                        v[4 * j + 2] = x[8 * c + j].z; v[4 * j + 3] = x[8 * c + j].w;
                    }
                    tmem_st32(tmem + lane_addr + kTmemQ + 64 * half + 32 * c, v);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kBarQFull));
        };
        TileWalk w;
        w.init(args.plan, grp);
        if (w.valid) load_q(w.seq * q_len + qi);
        if (threadIdx.x == 192) MLA_TRACE_POINT(3, kTraceProlog);
        for (int h = 0; w.valid && ok && !*abort_flag; ++h, w.advance()) {
            const int hb = h & 1;
            // ---- partial S(h) of this half, in log2 units, rounded to fp16
            if (!MLA_TW(kTwSFull, mbar_wait(bar(kBarSFull), h & 1))) { ok = false; break; }
            tc_fence_after();
            uint32_t own[32];
            {
                // both halves out of TMEM first, so that S(h+1) may start at once
                uint32_t va[32], vb[32];
                tmem_ld32(tmem + lane_addr + kTmemS, va);
                tmem_ld32(tmem + lane_addr + kTmemS + 32, vb);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kBarSFree));
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    own[j] = pack_f16(__uint_as_float(va[2 * j]) * sl2, __uint_as_float(va[2 * j + 1]) * sl2);
                    own[16 + j] = pack_f16(__uint_as_float(vb[2 * j]) * sl2, __uint_as_float(vb[2 * j + 1]) * sl2);
                }
                if (threadIdx.x == 192) MLA_TRACE_POINT(3, h);
            }
            // ---- publish: Own[hb] (read by our softmax warps and by the bulk copy
            // into the peer's X[hb]); both readers of tile h-2 must be done.
            if (h >= 2) {
                if (!MLA_TW(kTwOwnFree, mbar_wait(bar(kBarOwnFree0 + hb), ((h >> 1) - 1) & 1))) { ok = false; break; }
                if (!MLA_TW(kTwOwnFree, mbar_wait_cluster(bar(kBarXFree0 + hb), ((h >> 1) - 1) & 1))) { ok = false; break; }
            }
            const uint32_t own_buf = base + kOffOwn + hb * kXBytes;
#pragma unroll
            for (int c = 0; c < 8; ++c)
                st_shared_v4(own_buf + sw128(m, c), own[4 * c], own[4 * c + 1], own[4 * c + 2], own[4 * c + 3]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                const uint32_t off = quarter * 32 * 128;
                bulk_copy_s2s(x_peer + hb * kXBytes + off, own_buf + off, 32 * 128, xfull_peer + 8 * hb);
                mbar_arrive(bar(kBarOwnFull0 + hb));
            }
            // The peer's partial for tile h lands in our X[hb] (its phase h/2).
            if (threadIdx.x == 192) {
                mbar_arrive_expect_tx(bar(kBarXFull0 + hb), kXBytes);
                MLA_TRACE_POINT(4, h);
            }
            // S(h) was the last reader of this piece's Q-hat: load the next
            // piece's, after the partial is on its way (the next S waits for it,
            // the exchange of tile h does not).
            if (w.last()) {
                TileWalk nx = w;
                nx.advance();
                if (nx.valid) load_q(nx.seq * q_len + qi);
            }
        }
        if (!ok) *abort_flag = 1;
    } else {
        // ======================================================== softmax warps 2..5 and 12..15
        // Two warps per TMEM quarter: half kh takes keys 32kh..32kh+31 of each
        // score row and latent columns 128kh..128kh+127 of O; the pair agrees on
        // the row maximum through shared memory, meeting on named barrier
        // 1 + quarter.  Both warps walk the same tiles and meet at the same
        // points; a failed (timed-out) wait does not leave the loop at once: the
        // warp skips the tile's side effects up to the next meeting, where both
        // read each other's status and stop together (a hardware barrier has no
        // time limit, so neither may wait at one the other never reaches).
        const int kh = warp >= 12 ? 1 : 0;
        const uint32_t xfree_peer = mapa(bar(kBarXFree0), peer);
        float* red = reinterpret_cast<float*>(base_ptr + kOffRed);  // [2 tiles][2 halves][128 rows]
        volatile int* pair_ok = reinterpret_cast<volatile int*>(base_ptr + kOffFlags);
        bool ok = true;
        TileWalk w;
        w.init(args.plan, grp);
        float m_used = -CUDART_INF_F, l_part = 0.f;
        int n_keys = 0;
        for (int g = 0; w.valid; ++g, w.advance()) {
            const int b2 = g & 1;
            // ---- S(g) for this thread's 32 keys = own partial + the peer's (same order on both CTAs)
            if (ok) ok = MLA_TW(kTwXFull, mbar_wait(bar(kBarOwnFull0 + b2), (g >> 1) & 1));
            if (ok) ok = MLA_TW(kTwXFull, mbar_wait_cluster(bar(kBarXFull0 + b2), (g >> 1) & 1));
            float s[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) s[j] = 0.f;
            if (ok) {
                const uint32_t own_buf = base + kOffOwn + b2 * kXBytes;
                const uint32_t x_buf = base + kOffX + b2 * kXBytes;
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    const int c = 4 * kh + cc;
                    uint32_t a0, a1, a2, a3, o0, o1, o2, o3;
                    ld_shared_v4u(own_buf + sw128(m, c), a0, a1, a2, a3);
                    ld_shared_v4u(x_buf + sw128(m, c), o0, o1, o2, o3);
                    const uint32_t mine[4] = {a0, a1, a2, a3};
                    const uint32_t oth[4] = {o0, o1, o2, o3};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float2 v = sum_f16x2(mine[q], oth[q]);
                        s[8 * cc + 2 * q] = v.x;
                        s[8 * cc + 2 * q + 1] = v.y;
                    }
                }
            }
            // Both buffers are consumed (their values are in registers and used
            // by the adds above), so relaxed arrives suffice.
            __syncwarp();
            if (ok && lane == 0) {
                mbar_arrive(bar(kBarOwnFree0 + b2));
                mbar_arrive_remote_relaxed(xfree_peer + 8 * b2);
            }
            if (threadIdx.x == 64) MLA_TRACE_POINT(5, g);
            // ---- online softmax in base 2, lazy rescaling of O
            // query token qi of sequence b sees keys 0..T_b-q_len+qi
            if (w.first()) n_keys = args.seqlens[w.seq] - q_len + 1 + qi;
            const int key0 = w.t * kNk + 32 * kh;
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
            float* rg = red + (b2 * 2) * kHeads;  // this tile's [2 halves][128 rows]
            rg[kh * kHeads + m] = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
            volatile int* st_pair = pair_ok + (b2 * 4 + quarter) * 2;  // this tile's status of the pair
            if (lane == 0) st_pair[kh] = (ok && !*abort_flag) ? 1 : 0;
            named_bar_sync(1 + quarter, 64);
            if (!st_pair[0] || !st_pair[1]) {
                ok = false;
                break;
            }
            const float mx = fmaxf(rg[m], rg[kHeads + m]);
            if (threadIdx.x == 64) MLA_TRACE_POINT(8, g);
            const bool first = w.first();
            const bool grow = mx > m_used + 8.0f;  // rescale only when the max grows by > 2^8
            const float mb_new = grow ? mx : m_used;
            const float mb = (mb_new == -CUDART_INF_F) ? 0.f : mb_new;
            uint32_t pk[16];
            float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float p0 = ex2(s[2 * j] - mb), p1 = ex2(s[2 * j + 1] - mb);
                rs0 += p0;
                rs1 += p1;
                pk[j] = pack_bf16(p0, p1);
            }
            if (threadIdx.x == 64) MLA_TRACE_POINT(9, g);
            // P buffer b2 was last read by O(g-2).  (From here to the next
            // meeting a failed wait only skips work.)
            if (g >= 2 && ok) ok = MLA_TW(kTwPFree, mbar_wait(bar(kBarPFree0 + b2), ((g >> 1) - 1) & 1));
            if (grow && ok) {
                if (!first) {
                    // O must hold everything up to tile g-1 before it is rescaled.
                    ok = MLA_TW(kTwPFree, mbar_wait(bar(kBarPFree0 + (b2 ^ 1)), ((g - 1) >> 1) & 1));
                }
                if (ok && !first) {
                    tc_fence_after();
                    const float f = ex2(m_used - mx);
                    l_part *= f;
#pragma unroll 1
                    for (int c0 = 0; c0 < kHalfLat / 2; c0 += 32) {
                        uint32_t v[32];
                        tmem_ld32(tmem + lane_addr + kTmemO + 128 * kh + c0, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * f);
                        tmem_st32(tmem + lane_addr + kTmemO + 128 * kh + c0, v);
                    }
                }
                m_used = mx;
            }
            if (ok) {
                tc_fence_after();
                l_part += rs0 + rs1;
                tmem_st16(tmem + lane_addr + kTmemP + 32 * b2 + 16 * kh, pk);
                tmem_wait_st();
                tc_fence_before();
            }
            __syncwarp();
            if (ok && lane == 0) mbar_arrive(bar(kBarPFull0 + b2));
            if (threadIdx.x == 64) MLA_TRACE_POINT(6, g);
#ifndef MLA_TRACE_CYCLES
            if (threadIdx.x == 96) MLA_TRACE_POINT(11, g);
            if (threadIdx.x == 384) MLA_TRACE_POINT(12, g);
#endif
            if (threadIdx.x == 160) MLA_TRACE_POINT(13, g);
            // ---- epilogue at the end of a piece: this thread owns O row m, columns 128kh..+127
            float l_sum = 0.f;
            if (w.last()) {
                // the row's softmax denominator: both halves' partial sums
                float* rl = red + (b2 * 2) * kHeads;
                named_bar_sync(1 + quarter, 64);  // the pair has read this tile's maxima
                rl[kh * kHeads + m] = l_part;
                named_bar_sync(1 + quarter, 64);
                l_sum = rl[m] + rl[kHeads + m];
                if (ok) ok = mbar_wait(bar(kBarOFull), w.seg & 1);
            }
            if (w.last() && ok) {
                tc_fence_after();
                const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
                const int u = w.seq * q_len + qi;
                const int col0 = r * kHalfLat + 128 * kh;  // first latent column of this thread
                if (w.whole) {
                    __nv_bfloat16* dst = args.o_lat + ((size_t)u * kHeads + m) * kLat + col0;
#pragma unroll 1
                    for (int c0 = 0; c0 < kHalfLat / 2; c0 += 32) {
                        uint32_t v[32];
                        tmem_ld32(tmem + lane_addr + kTmemO + 128 * kh + c0, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 32; j += 16) {
                            uint32_t o[8];
#pragma unroll
                            for (int q = 0; q < 8; ++q)
                                o[q] = pack_bf16(__uint_as_float(v[j + 2 * q]) * inv, __uint_as_float(v[j + 2 * q + 1]) * inv);
                            if (args.o_lat_v8) {
                                st_global_v8(dst + c0 + j, o[0], o[1], o[2], o[3], o[4], o[5], o[6], o[7]);
                            } else {
                                *reinterpret_cast<uint4*>(dst + c0 + j) = make_uint4(o[0], o[1], o[2], o[3]);
                                *reinterpret_cast<uint4*>(dst + c0 + j + 8) = make_uint4(o[4], o[5], o[6], o[7]);
                            }
                        }
                    }
                } else {
                    // fp32 partial in column octets, [slot][c8][head][8]: a warp (32
                    // consecutive heads) writes 1 KB contiguous per octet (one 32-byte
                    // store per lane), and a consumer reading one head gets whole
                    // 32-byte sectors.
                    const size_t slot = (size_t)(grp + w.seq) * q_len + qi;
                    float* dst = args.part_o + (slot * (kLat / 8) * kHeads + m) * 8;
#pragma unroll 1
                    for (int c0 = 0; c0 < kHalfLat / 2; c0 += 32) {
                        uint32_t v[32];
                        tmem_ld32(tmem + lane_addr + kTmemO + 128 * kh + c0, v);
                        tmem_wait_ld();
                        const int o0 = (col0 + c0) / 8;
#pragma unroll
                        for (int j = 0; j < 32; j += 8) {
                            uint32_t o[8];
#pragma unroll
                            for (int q = 0; q < 8; ++q) o[q] = __float_as_uint(__uint_as_float(v[j + q]) * inv);
                            st_global_v8(dst + (size_t)(o0 + j / 8) * kHeads * 8, o[0], o[1], o[2], o[3], o[4], o[5],
                                         o[6], o[7]);
                        }
                    }
                    if (r == 0 && kh == 0)
                        args.part_lse[slot * kHeads + m] = l_sum > 0.f ? m_used + __log2f(l_sum) : -CUDART_INF_F;
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kBarOFree));
                if (threadIdx.x == 64) MLA_TRACE_POINT(7, g);
                if (threadIdx.x == 64) MLA_TRACE_POINT(5, kTraceProlog);
                if (threadIdx.x == 64) MLA_TRACE_ALL(4, global_timer_ns());
                m_used = -CUDART_INF_F;
                l_part = 0.f;
            }
        }
        if (!ok) *abort_flag = 1;
    }

#ifdef MLA_TRACE_WAITS
    if (threadIdx.x == 0 || threadIdx.x == 32 || threadIdx.x == 64 || threadIdx.x == 192 || threadIdx.x == 320) {
#pragma unroll
        for (int i = 0; i < kTwN; ++i)
            if (tw_acc[i]) MLA_TRACE_ALL(kTwBase + i, tw_acc[i]);
    }
#endif
    if (*abort_flag && threadIdx.x == 0) atomicOr(args.status, MLA_STATUS_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, kTmemCols);
    // The peer may still copy scores into this CTA's shared memory or arrive
    // on its barriers: neither CTA leaves before both are done.
    if (threadIdx.x == 0) MLA_TRACE_POINT(6, kTraceProlog);
    cluster_sync();
    if (threadIdx.x == 0) MLA_TRACE_POINT(7, kTraceProlog);
    if (threadIdx.x == 0) MLA_TRACE_ALL(5, global_timer_ns());
    MLA_KT(kKtAttend, 2);
}

// ------------------------------------------------------------------ plan

// Per sequence: cost_b = ceil(T_b / 64) + ovh (0 for an invalid length);
// prefix sums, the per-group share L = ceil(total / groups) (at least
// min_units), the list of sequences cut across groups, and o_lat = 0 for the
// tokens of sequences with an invalid length (their decode has no defined
// result).  One warp.
__device__ __forceinline__ void mla_plan_warp(const int32_t* __restrict__ seqlens, int B, int q_len, int T_max,
                                              int clusters, int ovh, int min_units, Plan* plan, int* status,
                                              __nv_bfloat16* o_lat, int lane) {
    int* gfirst = reinterpret_cast<int*>(plan + 1);
    int* pre = gfirst + kPlanMaxGroups;
    int* splits = pre + B + 1;
    const int groups = clusters / q_len > 0 ? clusters / q_len : 1;
    for (int g = lane; g < groups; g += 32) gfirst[g] = B;
    int carry = 0, c_min = INT_MAX, c_max = 0;
    if (lane == 0) pre[0] = 0;
    for (int base = 0; base < B; base += 32) {
        const int b = base + lane;
        int c = 0;
        if (b < B) {
            const int T = seqlens[b];
            if (T < q_len || T > T_max) atomicOr(status, MLA_STATUS_BAD_SEQLEN);
            else c = (T + kNk - 1) / kNk + ovh;
            c_min = min(c_min, c);
            c_max = max(c_max, c);
        }
        int v = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += y;
        }
        if (b < B) pre[b + 1] = carry + v;
        carry += __shfl_sync(0xffffffffu, v, 31);
    }
    int L = (carry + groups - 1) / groups;
    // A batch of equal, valid lengths may be cut at sequence boundaries
    // instead: no partials and no combine pass, which costs more than a few
    // tiles per group; taken when the whole-sequence share is within a quarter
    // of the even share.
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        c_min = min(c_min, __shfl_xor_sync(0xffffffffu, c_min, o));
        c_max = max(c_max, __shfl_xor_sync(0xffffffffu, c_max, o));
    }
    if (c_min == c_max && c_max > 0) {
        const int whole = ((B + groups - 1) / groups) * c_max;
        if (whole <= L + L / 4) L = whole;
    }
    if (L < min_units) L = min_units;
    if (L < 1) L = 1;
    __syncwarp();
    int n_split = 0;
    for (int base = 0; base < B; base += 32) {
        const int b = base + lane;
        bool split = false, invalid = false;
        if (b < B) {
            const int lo = pre[b], hi = pre[b + 1];
            if (hi == lo) invalid = true;
            else split = (lo + ovh) / L != (hi - 1) / L;
            // groups whose first cost unit g L falls in [lo, hi) start in sequence b
            if (hi > lo)
                for (int g = (lo + L - 1) / L; g <= (hi - 1) / L && g < groups; ++g) gfirst[g] = b;
        }
        const unsigned msk = __ballot_sync(0xffffffffu, split);
        if (split) splits[n_split + __popc(msk & ((1u << lane) - 1))] = b;
        n_split += __popc(msk);
        unsigned inv = __ballot_sync(0xffffffffu, invalid);
        while (inv) {
            const int bi = base + __ffs(inv) - 1;
            inv &= inv - 1;
            uint4* dst = reinterpret_cast<uint4*>(o_lat + (size_t)bi * q_len * kHeads * kLat);
            for (int i = lane; i < q_len * kHeads * kLat / 8; i += 32) dst[i] = make_uint4(0, 0, 0, 0);
        }
    }
    if (lane == 0) {
        plan->L = L;
        plan->ovh = ovh;
        plan->B = B;
        plan->total = carry;
        plan->n_split = n_split;
        plan->q_len = q_len;
        plan->groups = groups;
    }
}

__global__ void __launch_bounds__(32) mla_plan_kernel(const int32_t* __restrict__ seqlens, int B, int q_len,
                                                      int T_max, int clusters, int ovh, int min_units, Plan* plan,
                                                      int* status, __nv_bfloat16* o_lat) {
    mla_plan_warp(seqlens, B, q_len, T_max, clusters, ovh, min_units, plan, status, o_lat, threadIdx.x);
}

// ------------------------------------------------------------------ combine

// The pieces of query token qi of sequence b: groups p_lo..p_hi, piece p
// stored in partial slot (p + b) * q_len + qi if its clip of the sequence's
// tiles is non-empty.  split = false when one group holds the whole
// sequence (o_lat was then written directly, or zeroed for an invalid
// length).
struct UnitPieces {
    int p_lo, p_hi, c_lo, tiles, L, ovh;
    bool split;
    __device__ void init(const Plan* plan, int b) {
        const int* pre = plan_prefix(plan);
        L = plan->L;
        ovh = plan->ovh;
        c_lo = pre[b];
        const int c_hi = pre[b + 1];
        tiles = c_hi > c_lo ? c_hi - c_lo - ovh : 0;
        p_lo = c_lo / L;
        p_hi = c_hi > c_lo ? (c_hi - 1) / L : p_lo;
        split = c_hi > c_lo && (c_lo + ovh) / L != (c_hi - 1) / L;
    }
    // Group p holds tiles [p L - c_lo - ovh, (p+1) L - c_lo - ovh) of the
    // sequence, clipped to [0, tiles); an empty clip wrote no partial.
    __device__ bool nonempty(int p) const {
        int s0 = p * L - c_lo - ovh, e0 = (p + 1) * L - c_lo - ovh;
        s0 = s0 < 0 ? 0 : (s0 > tiles ? tiles : s0);
        e0 = e0 < 0 ? 0 : (e0 > tiles ? tiles : e0);
        return e0 > s0;
    }
};

// Running merge state of split partials for one (unit, head), lane l
// holding columns 4(l + 32 j) .. +3, j = 0..3: max m of the pieces' base-2
// LSEs, sum of 2^(lse - m), and sum of 2^(lse - m) o_p (the softmax of the
// pieces' log-sum-exps, unnormalised).
struct MergeState {
    float m, wsum;
    float4 acc[4];
    __device__ void clear() {
        m = -CUDART_INF_F;
        wsum = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    // Folds in another state (m2, w2, a2).
    __device__ void fold(float m2, float w2, const float4 (&a2)[4]) {
        const float mb = fmaxf(m, m2);
        if (mb == -CUDART_INF_F) return;
        const float r0 = exp2f(m - mb), r1 = exp2f(m2 - mb);  // -inf gives 0
        wsum = wsum * r0 + w2 * r1;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            acc[j].x = acc[j].x * r0 + a2[j].x * r1; acc[j].y = acc[j].y * r0 + a2[j].y * r1;
            acc[j].z = acc[j].z * r0 + a2[j].z * r1; acc[j].w = acc[j].w * r0 + a2[j].w * r1;
        }
        m = mb;
    }
    __device__ void normalise() {
        const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            acc[j].x *= inv; acc[j].y *= inv; acc[j].z *= inv; acc[j].w *= inv;
        }
    }
};

// Adds pieces p_lo + first, p_lo + first + step, ... of one (unit, head) to
// `st` (one warp); pieces are read four at a time so that their loads
// overlap.
__device__ __forceinline__ void merge_pieces_warp(const UnitPieces& up, int b, int qi, int q_len, int h,
                                                  const float* __restrict__ part_o,
                                                  const float* __restrict__ part_lse, int lane, int first, int step,
                                                  MergeState& st) {
    for (int p0 = up.p_lo + first; p0 <= up.p_hi; p0 += 4 * step) {
        float lse[4];
        float4 v[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int p = p0 + i * step;
            lse[i] = -CUDART_INF_F;
            if (p <= up.p_hi && up.nonempty(p)) {
                const size_t slot = (size_t)(p + b) * q_len + qi;
                lse[i] = __ldg(part_lse + slot * kHeads + h);
                // columns 4q..4q+3, q = lane + 32 j: octet q / 2, half q % 2
                const float4* src = reinterpret_cast<const float4*>(part_o) + (slot * (kLat / 8) * kHeads + h) * 2;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int q = lane + 32 * j;
                    v[i][j] = __ldg(src + (size_t)(q / 2) * kHeads * 2 + (q % 2));
                }
            } else {
#pragma unroll
                for (int j = 0; j < 4; ++j) v[i][j] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) st.fold(lse[i], lse[i] == -CUDART_INF_F ? 0.f : 1.f, v[i]);
    }
}

// Split combine as its own step: one warp per (split unit, head), eight
// heads per CTA; writes o_lat (bf16) of the split units.
__global__ void __launch_bounds__(256) mla_combine_kernel(const Plan* __restrict__ plan,
                                                          const float* __restrict__ part_o,
                                                          const float* __restrict__ part_lse,
                                                          __nv_bfloat16* __restrict__ o_lat) {
    MLA_KT(kKtCombine, 0);
    pdl_wait();
    pdl_trigger();
    MLA_KT(kKtCombine, 1);
    const int q_len = plan->q_len;
    const int work = blockIdx.x / (kHeads / 8);
    if (work >= plan->n_split * q_len) {
        MLA_KT(kKtCombine, 2);
        return;
    }
    const int lane = threadIdx.x % 32;
    const int h = (blockIdx.x % (kHeads / 8)) * 8 + threadIdx.x / 32;
    const int b = plan_splits(plan)[work / q_len];
    const int qi = work % q_len;
    UnitPieces up;
    up.init(plan, b);
    MergeState ms;
    ms.clear();
    merge_pieces_warp(up, b, qi, q_len, h, part_o, part_lse, lane, 0, 1, ms);
    ms.normalise();
    uint2* dst = reinterpret_cast<uint2*>(o_lat + ((size_t)(b * q_len + qi) * kHeads + h) * kLat) + lane;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint2 o;
        o.x = pack_bf16(ms.acc[j].x, ms.acc[j].y);
        o.y = pack_bf16(ms.acc[j].z, ms.acc[j].w);
        dst[32 * j] = o;
    }
    MLA_KT(kKtCombine, 2);
}

}  // namespace sm100
}  // namespace mla
