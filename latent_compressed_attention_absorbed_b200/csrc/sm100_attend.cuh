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
// Work split.  One query token's 128 heads are the M dimension of every
// MMA.  Its fp32 output accumulator, 128 heads x 512 latent columns, fills
// the 512 TMEM columns of an SM, so a cluster of two CTAs shares the work:
//   * the scoring CTA (rank 0) holds Q-hat (576 bf16 per head) in TMEM,
//     loads whole cache rows (576 columns) for 64 keys at a time and computes
//     the exact fp32 scores S (36 MMAs of K = 16 into one of two TMEM
//     buffers), runs the online softmax, and streams P (bf16) and each row's
//     rescale factor and running sum to the accumulating CTA: the softmax
//     warps write them into a local staging slot and one lane per TMEM
//     quarter bulk-copies the quarter's rows into the peer's slot;
//   * the accumulating CTA (rank 1) loads the latent part of the same rows
//     (an L2 hit) and accumulates O += P . C_KV with P as the shared-memory
//     A operand (two MMAs of N = 256 per K step), rescales O's rows when the
//     scorer's running maximum grew, and writes the normalised o_lat or the
//     split partial at the end of a piece.
// The traffic between the pair is one way (18 KB per 64 keys) through a
// ring of three slots, so its latency is hidden; the scorer's stage is
// released as soon as its score MMAs complete.
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
// Roles (512 threads; warp w reaches TMEM lanes 32*(w%4)..+31, and lane l
// of a warp owns head 32*(w%4)+l, a whole row):
//   scorer:      warp 0 TMA producer; warp 1 TMEM owner and S issuer;
//                warps 2-5 and 12-15 softmax, two per TMEM quarter (32 keys
//                each); warps 6-9 load Q-hat into TMEM once per piece;
//   accumulator: warp 0 TMA producer; warp 1 TMEM owner and O issuer;
//                warps 2-5 and 12-15 rescale / epilogue, two per quarter
//                (256 columns each); warp 10 returns consumed P slots.
// Every wait is bounded; on expiry the kernel flags MLA_STATUS_TIMEOUT,
// stops issuing work, drains what it has in flight (stage loads, MMAs, the
// peer's copies into its shared memory) and tears down normally (the two
// softmax warps of a quarter, which meet on a named barrier, decide together
// whether to stop, so neither is left waiting).
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

// Shared-memory map (offsets from a 1024-aligned base).
// Scoring CTA (cluster rank 0):
//   stages:  kSStages whole cache rows of 64 keys: 9 SW128 chunks of 64 keys
//            x 64 columns (latent 0..511, then RoPE 512..575), 72 KB each;
//   staging: kPSlots local copies of the accumulator's P slots (same layout),
//            written by the softmax warps and bulk-copied to the peer;
//   red, flags: the softmax pairs' row maxima / sums and their status;
//   qstage:  per TMEM quarter, one 128-byte column block of its 32 Q-hat rows
//            (the Q-hat loaders read rows coalesced and transpose them here).
// Accumulating CTA (cluster rank 1):
//   vstages: kVStages latent parts of 64 keys (8 SW128 chunks), 64 KB each;
//   pslots:  kPSlots slots, each P of 128 heads x 64 keys as two matrices of
//            32 keys (bf16, 64-byte rows, SW64, K-major: the A operand of the
//            O MMA's first and last two K steps), then per key half and head
//            8 bytes: the rescale factor of O and that half's sum of p.
constexpr int kChunk = kNk * 128;            // 8192: 64 keys x 64 columns
constexpr int kSStages = 2;
constexpr int kSStageBytes = 9 * kChunk;     // 73728
constexpr int kVStages = 2;
constexpr int kVStageBytes = 8 * kChunk;     // 65536
constexpr int kPSlots = 3;
constexpr int kPHalf = kHeads * 64;          // 8192: one key half of P
constexpr int kPData = 2 * kPHalf;           // 16384
constexpr int kPSlotBytes = kPData + 2 * kHeads * 8;  // 18432
constexpr int kOffSStages = 0;
constexpr int kOffStaging = kSStages * kSStageBytes;
constexpr int kOffRed = kOffStaging + kPSlots * kPSlotBytes;  // [2 tiles][2 halves][128 rows] fp32
constexpr int kOffFlags = kOffRed + 2 * 2 * kHeads * 4;       // [2 tiles][4 quarters][2] int
constexpr int kOffQStage = (kOffFlags + 2 * 4 * 2 * 4 + 127) & ~127;  // [4 quarters][32 rows][128 B]: Q-hat transpose
constexpr int kScorerEnd = kOffQStage + 4 * 32 * 128;
#ifndef MLA_SCORE_PREFETCH
#define MLA_SCORE_PREFETCH 0
#endif
// Row tiles the scorer prefetches into L2 ahead of its stage loads (0: off;
// 4 and 8 tiles measured slower than none on B200, where the two-stage ring
// of each scorer already keeps HBM busy).
constexpr int kScorePrefetch = MLA_SCORE_PREFETCH;
constexpr int kOffVStages = 0;
constexpr int kOffPSlots = kVStages * kVStageBytes;
constexpr int kAccumEnd = kOffPSlots + kPSlots * kPSlotBytes;
constexpr int kOffBars = (kScorerEnd > kAccumEnd ? kScorerEnd : kAccumEnd);
constexpr int kBarBytes = 512;  // barrier block: the mbarriers, then the TMEM base and the abort flag
constexpr int kAttSmem = kOffBars + kBarBytes + 1024;
static_assert(kOffPSlots % 1024 == 0 && kPSlotBytes % 1024 == 0, "P slots must start on 1024-byte boundaries");
static_assert(kAttSmem <= 232448, "attention kernel shared memory exceeds 227 KB");

// Tensor-memory maps: 512 columns of 32 bits, lane = head.
constexpr int kTmemCols = 512;
constexpr int kTmemQ = 0;    // scorer: Q-hat, 576 bf16, two per column (288 columns)
constexpr int kTmemS = 384;  // scorer: two S buffers of 64 fp32 columns (384, 448)
constexpr int kTmemO = 0;    // accumulator: O, 512 fp32 latent columns
constexpr int kAttThreads = 512;

// Barrier indices (8 bytes each) inside the barrier block.
enum {
    // scorer
    kBarFull0 = 0,                      // stage loaded (tx)
    kBarEmpty0 = kBarFull0 + kSStages,  // stage read by S (MMA commit)
    kBarSFull0 = kBarEmpty0 + kSStages, // S(g) in buffer g%2 (MMA commit)
    kBarSFree0 = kBarSFull0 + 2,        // S buffer read by the 8 softmax warps
    kBarQFull = kBarSFree0 + 2,         // Q-hat of a piece in TMEM (4 loader warps)
    kBarQRead,                          // the last S of a piece complete: Q-hat may be replaced (MMA commit)
    kBarSlotFree0 = kBarQRead + 1,      // accumulator's P slot consumed (remote arrive)
    // accumulator
    kBarVFull0 = kBarSlotFree0 + kPSlots,  // latent part loaded (tx)
    kBarVEmpty0 = kBarVFull0 + kVStages,   // latent part read by O (MMA commit)
    kBarPFull0 = kBarVEmpty0 + kVStages,   // P(g) and its row data landed (tx, from the scorer)
    kBarPDone0 = kBarPFull0 + kPSlots,     // O(g) complete: the slot was read (MMA commit)
    kBarRescaled0 = kBarPDone0 + kPSlots,  // O rows rescaled for tile g if needed (8 epilogue warps)
    kBarOFull = kBarRescaled0 + kPSlots,   // last O of a piece complete (MMA commit)
    kBarOFree,                             // O read by the epilogue (8 warps)
    // both
    kBarDrain,                             // every MMA of the issuer complete (teardown)
    kNumBars
};
static_assert(8 * (kNumBars + 2) <= kBarBytes, "barrier block too small");

// Optional timing trace (compile with -DMLA_TRACE): global-timer stamps (ns)
// of both CTAs of one cluster at fixed points of every tile, read back by
// mla_trace_read.  Scorer: 0 stage loads issued, 6 stage landed (seen by
// the S issuer), 14 S issue start, 1 S issued, 12 S complete (seen by a
// softmax warp), 3 / 13 S read by the two softmax warps of quarter 2, 8 row
// maximum agreed, 9 P computed, 10 slot free, 4 P handed to the bulk copies.
// Accumulator: 0 stage loads issued, 5 O rows rescaled (or checked), 15 O
// issue start, 2 O issued, 7 piece epilogue done.
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
    kTwFull,      // S issuer: stage loaded / O issuer: latent part loaded
    kTwSFree,     // S issuer: S buffer read out of TMEM
    kTwQFull,     // S issuer: Q-hat of a piece
    kTwSFull,     // (unused)
    kTwOwnFree,   // (unused)
    kTwXFull,     // softmax: S complete / epilogue: P slot landed
    kTwPFree,     // softmax: the peer's P slot consumed
    kTwPFull,     // O issuer: P slot landed, rows rescaled
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
    uint64_t wait_limit_ns;       // time limit of every barrier wait
    int withhold_tile;            // test hook (>= 0): the loaders stop before this tile (see mla.h)
    const uint8_t* cache;         // the cache rows, for the L2 prefetch of whole row tiles
    int64_t stride_b, stride_t;   // (bytes; the prefetch runs only when a tile's rows are contiguous)
    int T_max;
};

// Byte offset of 16-byte chunk c of row r in a buffer of 128-byte rows whose
// chunks are permuted by row (c ^ (r % 8)): the SW128 layout the tensor core
// reads (K-major, 1024-byte groups of 8 rows), and the 8 rows a quarter-warp
// touches at once land in 8 different bank groups.
__device__ __forceinline__ uint32_t sw128(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }
// The same for 64-byte rows (SW64: chunk c of row r moves to c ^ ((r / 2) % 4)).
__device__ __forceinline__ uint32_t sw64(int r, int c) { return (uint32_t)(r * 64 + ((c ^ ((r >> 1) & 3)) << 4)); }

// Rows at or beyond the sequence length hold no cached token: zero `nchunks`
// SW128 chunks of 64 keys from row r0 on (one warp), so that masked rows can
// inject no NaN / Inf through p = 0.
__device__ __forceinline__ void zero_rows(uint32_t tile, int nchunks, int r0, int lane) {
    for (int row = r0 + (lane >> 3); row < kNk; row += 4)
        for (int c = 0; c < nchunks; ++c) st_shared_v4(tile + c * kChunk + row * 128 + (lane & 7) * 16, 0, 0, 0, 0);
    fence_proxy_async_smem();
}

// mapRow: the cache [B][T_max][576] bf16, box 64 columns x 64 keys, SW128.
__global__ void __launch_bounds__(kAttThreads, 1)
    mla_attend_kernel(const __grid_constant__ CUtensorMap mapRow, AttendArgs args) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* base_ptr = smem_raw + (base - raw);
    auto bar = [&](int i) { return base + kOffBars + 8u * i; };
    const uint32_t tmem_slot = bar(kNumBars);
    const uint32_t abort_addr = bar(kNumBars + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(base_ptr + kOffBars + 8 * (kNumBars + 1));
    const uint64_t lim = args.wait_limit_ns;

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const uint32_t rank = cluster_ctarank() & 1;  // 0: scorer, 1: accumulator
    const uint32_t peer = rank ^ 1;
    const int cl = (int)cluster_id_x();
    const int q_len = args.q_len;
    const int grp = cl / q_len, qi = cl % q_len;
    [[maybe_unused]] const uint32_t r = rank;  // for the trace macros

    if (threadIdx.x == 0) MLA_TRACE_POINT(0, kTraceProlog);
    if (threadIdx.x == 0) MLA_TRACE_ALL(0, global_timer_ns());
    MLA_KT(kKtAttend, 0);
#ifdef MLA_TRACE_WAITS
    unsigned long long tw_acc[kTwN];
#pragma unroll
    for (int i = 0; i < kTwN; ++i) tw_acc[i] = 0;
#endif
    if (threadIdx.x == 0) {
        if (rank == 0) {
            for (int s = 0; s < kSStages; ++s) {
                mbar_init(bar(kBarFull0 + s), 1);
                mbar_init(bar(kBarEmpty0 + s), 1);
            }
            for (int s = 0; s < 2; ++s) {
                mbar_init(bar(kBarSFull0 + s), 1);
                mbar_init(bar(kBarSFree0 + s), 8);
            }
            mbar_init(bar(kBarQFull), 4);
            mbar_init(bar(kBarQRead), 1);
            for (int s = 0; s < kPSlots; ++s) mbar_init(bar(kBarSlotFree0 + s), 1);
        } else {
            for (int s = 0; s < kVStages; ++s) {
                mbar_init(bar(kBarVFull0 + s), 1);
                mbar_init(bar(kBarVEmpty0 + s), 1);
            }
            for (int s = 0; s < kPSlots; ++s) {
                mbar_init(bar(kBarPFull0 + s), 1);
                mbar_init(bar(kBarPDone0 + s), 1);
                mbar_init(bar(kBarRescaled0 + s), 8);
            }
            mbar_init(bar(kBarOFull), 1);
            mbar_init(bar(kBarOFree), 8);
        }
        mbar_init(bar(kBarDrain), 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&mapRow);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    // The peer's barriers must be initialised before any remote access.
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(base_ptr + kOffBars + 8 * kNumBars);
    // The set-up above overlaps the previous kernel; the plan, Q-hat and the
    // cache are read only once it has completed.
    pdl_wait();
    if (threadIdx.x == 0) pdl_trigger();
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
    const int m = quarter * 32 + lane;                          // head / TMEM lane
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;  // the warp's TMEM subpartition
    const bool softmax_warp = (warp >= 2 && warp <= 5) || warp >= 12;
    const int kh = warp >= 12 ? 1 : 0;  // key half (scorer) / column half (accumulator)
    int n_loads = 0;                    // stage loads issued (producer lane), for the teardown

    if (!active) {
        // idle cluster (the cluster count is not a multiple of q_len)
    } else if (warp == 0) {
        // ======================================================== TMA producer (both CTAs)
        // scorer: whole rows (9 chunks) into kSStages stages, released by S;
        // accumulator: latent parts (8 chunks) into kVStages stages, released by O.
        if (lane == 0) {
            const int nst = rank == 0 ? kSStages : kVStages;
            const int nch = rank == 0 ? 9 : 8;
            const int sbytes = rank == 0 ? kSStageBytes : kVStageBytes;
            const int full0 = rank == 0 ? kBarFull0 : kBarVFull0;
            const int empty0 = rank == 0 ? kBarEmpty0 : kBarVEmpty0;
            TileWalk w, wp;
            w.init(args.plan, grp);
            wp = w;
            // The scorer prefetches whole row tiles into L2 a few tiles ahead
            // of its stage loads (a tile is contiguous when rows are packed);
            // the accumulator's loads of the same tiles then hit L2.
            const bool pf = rank == 0 && kScorePrefetch > 0 && args.stride_t == (int64_t)kRow * 2;
            auto prefetch_tile = [&](const TileWalk& t) {
                const int rows = args.T_max - t.t * kNk < kNk ? args.T_max - t.t * kNk : kNk;
                if (rows > 0)
                    prefetch_l2_bulk(args.cache + (size_t)t.seq * args.stride_b + (size_t)t.t * kNk * args.stride_t,
                                     (uint32_t)rows * kRow * 2);
            };
            if (pf)
                for (int i = 0; i < kScorePrefetch && wp.valid; ++i, wp.advance()) prefetch_tile(wp);
            for (int n = 0; w.valid && !*abort_flag; ++n, w.advance()) {
                // Test hook: stop before tile `withhold_tile`, which is then never
                // loaded, so that a bounded wait for it runs out.
                if (n == args.withhold_tile) break;
                if (pf && wp.valid) {
                    prefetch_tile(wp);
                    wp.advance();
                }
                const int st = n % nst;
                if (n >= nst && !MLA_TW(kTwEmpty, mbar_wait(bar(empty0 + st), ((n / nst) - 1) & 1, lim))) {
                    *abort_flag = 1;
                    break;
                }
                const uint32_t dst = base + st * sbytes;
                mbar_arrive_expect_tx(bar(full0 + st), sbytes);
                for (int c = 0; c < nch; ++c) tma_load_3d(dst + c * kChunk, &mapRow, bar(full0 + st), 64 * c, w.t * kNk, w.seq);
                n_loads = n + 1;
                MLA_TRACE_POINT(0, n);
            }
        }
    } else if (rank == 0 && warp == 1) {
        // ======================================================== scorer: S issuer (whole warp waits, lane 0 issues)
        // S(g) = Q-hat . row^T over all 576 columns (36 MMAs of K = 16, Q-hat
        // from TMEM) into buffer g%2; the stage is released as soon as S(g)
        // completes.
        constexpr uint32_t idS = idesc_bf16_f32(kHeads, kNk, false, false);
        const uint64_t dRowK = smem_desc(base + kOffSStages, 16, 1024, kSw128);  // cache rows, K-major
        TileWalk ws;
        ws.init(args.plan, grp);
        int T_s = ws.valid ? args.seqlens[ws.seq] : 0;  // length of the sequence of tile g
        bool ok = true;
        for (int g = 0; ws.valid && ok && !*abort_flag; ++g) {
            const int sb = g & 1, st = g % kSStages;
            if (ws.first() && !MLA_TW(kTwQFull, warp_wait(bar(kBarQFull), ws.seg & 1, lim))) { ok = false; break; }
            if (!MLA_TW(kTwFull, warp_wait(bar(kBarFull0 + st), (g / kSStages) & 1, lim))) { ok = false; break; }
            if (lane == 0) MLA_TRACE_POINT(6, g);
            if (g >= 2 && !MLA_TW(kTwSFree, warp_wait(bar(kBarSFree0 + sb), ((g >> 1) - 1) & 1, lim))) { ok = false; break; }
            const uint32_t tile = base + kOffSStages + st * kSStageBytes;
            const int valid = T_s - ws.t * kNk;
            if (valid < kNk) zero_rows(tile, 9, valid < 0 ? 0 : valid, lane);
            __syncwarp();
            tc_fence_after();
            if (lane == 0) {
                MLA_TRACE_POINT(14, g);
                const uint32_t dS = tmem + kTmemS + 64 * sb;
                const uint64_t dB = dRowK + ((st * kSStageBytes) >> 4);
#pragma unroll
                for (int k = 0; k < 36; ++k)
                    mma_f16_ts(dS, tmem + kTmemQ + 8 * k, dB + (((k >> 2) * kChunk + 32 * (k & 3)) >> 4), idS, k ? 1u : 0u);
                mma_commit(bar(kBarSFull0 + sb));
                mma_commit(bar(kBarEmpty0 + st));
                if (ws.last()) mma_commit(bar(kBarQRead));
                MLA_TRACE_POINT(1, g);
            }
            __syncwarp();
            const int seq_before = ws.seq;
            ws.advance();
            if (ws.valid && ws.seq != seq_before) T_s = args.seqlens[ws.seq];
        }
        if (!ok) *abort_flag = 1;
    } else if (rank == 0 && warp >= 6 && warp <= 9) {
        // ======================================================== scorer: Q-hat loaders
        // Row m's 576 Q-hat values -> TMEM columns 0..287 (this thread), once
        // per piece; the next piece's Q-hat goes in after the last S of the
        // current piece has completed (S reads Q-hat from TMEM), which the S
        // issuer signals on its own barrier, one phase per piece: the loaders
        // are never more than one phase behind it.
        bool ok = true;
        // Rows are read coalesced (a warp instruction covers four whole 128-byte
        // row blocks), staged in shared memory with the 16-byte pieces of row r
        // permuted by r % 8, and read back one row per lane for tcgen05.st;
        // the next column block's loads are in flight during the transpose.
        const uint32_t qbuf = base + kOffQStage + quarter * 32 * 128;
        const int rr = lane >> 3, pc = lane & 7;  // this lane's row within a group of four, and 16-byte piece
        auto load_q = [&](int u) {
            const uint4* src = reinterpret_cast<const uint4*>(args.q_hat + ((size_t)u * kHeads + quarter * 32) * kRow);
            uint4 cur[8], nxt[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) cur[j] = __ldg(src + (size_t)(4 * j + rr) * (kRow / 8) + pc);
#pragma unroll 1
            for (int c = 0; c < 9; ++c) {
                if (c + 1 < 9) {
#pragma unroll
                    for (int j = 0; j < 8; ++j) nxt[j] = __ldg(src + (size_t)(4 * j + rr) * (kRow / 8) + 8 * (c + 1) + pc);
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int row = 4 * j + rr;
                    st_shared_v4(qbuf + row * 128 + ((pc ^ (row & 7)) << 4), cur[j].x, cur[j].y, cur[j].z, cur[j].w);
                }
                __syncwarp();
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t v[16];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int piece = 4 * h + q;
                        ld_shared_v4u(qbuf + lane * 128 + ((piece ^ (lane & 7)) << 4), v[4 * q], v[4 * q + 1], v[4 * q + 2],
                                      v[4 * q + 3]);
                    }
                    tmem_st16(tmem + lane_addr + kTmemQ + 32 * c + 16 * h, v);
                }
                __syncwarp();  // the buffer is rewritten for the next block
#pragma unroll
                for (int j = 0; j < 8; ++j) cur[j] = nxt[j];
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kBarQFull));
        };
        TileWalk w;
        w.init(args.plan, grp);
        if (w.valid) load_q(w.seq * q_len + qi);
        for (; w.valid && ok && !*abort_flag; w.advance()) {
            if (!w.last()) continue;
            TileWalk nx = w;
            nx.advance();
            if (!nx.valid) break;
            // every S of piece w.seg has read Q-hat
            if (!warp_wait(bar(kBarQRead), w.seg & 1, lim)) { ok = false; break; }
            tc_fence_after();
            load_q(nx.seq * q_len + qi);
        }
        if (!ok) *abort_flag = 1;
    } else if (rank == 0 && softmax_warp) {
        // ======================================================== scorer: softmax warps 2..5 and 12..15
        // Two warps per TMEM quarter: half kh takes keys 32kh..32kh+31 of each
        // score row; the pair agrees on the row maximum through shared memory,
        // meeting on named barrier 1 + quarter.  Both warps walk the same tiles
        // and meet at the same points; a failed (timed-out) wait does not leave
        // the loop at once: the warp skips the tile's side effects up to the
        // next meeting, where both read each other's status and stop together.
        // P goes to the accumulator's slot g % kPSlots with st.async (SW128
        // rows, the O MMA's A operand), with this row's rescale factor of O
        // and the half's running sum of p.
        const uint32_t pslot_peer = mapa(base + kOffPSlots, peer);
        const uint32_t pfull_peer = mapa(bar(kBarPFull0), peer);
        float* red = reinterpret_cast<float*>(base_ptr + kOffRed);  // [2 tiles][2 halves][128 rows]
        volatile int* pair_ok = reinterpret_cast<volatile int*>(base_ptr + kOffFlags);
        const float sl2 = args.scale_log2;
        bool ok = true;
        TileWalk w;
        w.init(args.plan, grp);
        float m_used = -CUDART_INF_F, l_part = 0.f;
        int n_keys = 0;
        for (int g = 0; w.valid; ++g, w.advance()) {
            const int sb = g & 1, b2 = g & 1, slot = g % kPSlots;
            if (ok) ok = MLA_TW(kTwXFull, warp_wait(bar(kBarSFull0 + sb), (g >> 1) & 1, lim));
            if (threadIdx.x == 64) MLA_TRACE_POINT(12, g);
            float s[32];
            if (ok) {
                tc_fence_after();
                uint32_t v[32];
                tmem_ld32(tmem + lane_addr + kTmemS + 64 * sb + 32 * kh, v);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) s[j] = __uint_as_float(v[j]) * sl2;
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) s[j] = 0.f;
            }
            tc_fence_before();
            __syncwarp();
            if (ok && lane == 0) mbar_arrive(bar(kBarSFree0 + sb));
            if (threadIdx.x == 64) MLA_TRACE_POINT(3, g);
            if (threadIdx.x == 448) MLA_TRACE_POINT(13, g);
            // ---- online softmax in base 2; O (in the accumulator) is rescaled
            // lazily, only when the row maximum grows by more than 2^8.
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
            const bool grow = mx > m_used + 8.0f;
            float f = 1.0f;  // factor the accumulator applies to O's row before adding P(g)
            if (grow) {
                if (!first) {
                    f = ex2(m_used - mx);
                    l_part *= f;
                }
                m_used = mx;
            }
            const float mb = (m_used == -CUDART_INF_F) ? 0.f : m_used;
            uint32_t pk[16];
            float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float p0 = ex2(s[2 * j] - mb), p1 = ex2(s[2 * j + 1] - mb);
                rs0 += p0;
                rs1 += p1;
                pk[j] = pack_bf16(p0, p1);
            }
            l_part += rs0 + rs1;
            if (threadIdx.x == 64) MLA_TRACE_POINT(9, g);
            // ---- send P(g): the accumulator must have consumed slot g%kPSlots
            // (tile g - kPSlots), which also means the bulk copies that read
            // the local staging slot have completed.  This warp's half rows
            // are a contiguous 2 KB of its key half's matrix (and 256 bytes
            // of row data), so it copies them to the peer itself.
            // (from here to the next meeting a failed wait only skips work)
            if (ok && g >= kPSlots)
                ok = MLA_TW(kTwPFree, warp_wait_cluster(bar(kBarSlotFree0 + slot), ((g / kPSlots) - 1) & 1, lim));
            if (threadIdx.x == 64) MLA_TRACE_POINT(10, g);
            if (ok) {
                const uint32_t stg = base + kOffStaging + slot * kPSlotBytes;
#pragma unroll
                for (int cc = 0; cc < 4; ++cc)
                    st_shared_v4(stg + kPHalf * kh + sw64(m, cc), pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
                st_shared_v2(stg + kPData + 1024 * kh + 8 * m, __float_as_uint(f), __float_as_uint(l_part));
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    const uint32_t dst = pslot_peer + slot * kPSlotBytes;
                    const uint32_t pb = pfull_peer + 8 * slot;
                    const uint32_t po = kPHalf * kh + quarter * 32 * 64, ao = kPData + 1024 * kh + quarter * 32 * 8;
                    bulk_copy_s2s(dst + po, stg + po, 32 * 64, pb);
                    bulk_copy_s2s(dst + ao, stg + ao, 32 * 8, pb);
                }
            }
            if (threadIdx.x == 64) MLA_TRACE_POINT(4, g);
            // ---- end of a piece: the LSE of a split piece (base 2), from both halves' sums
            if (w.last()) {
                float* rl = red + (b2 * 2) * kHeads;
                named_bar_sync(1 + quarter, 64);  // the pair has read this tile's maxima
                rl[kh * kHeads + m] = l_part;
                named_bar_sync(1 + quarter, 64);
                const float l_sum = rl[m] + rl[kHeads + m];
                if (ok && !w.whole && kh == 0) {
                    const size_t pslot = (size_t)(grp + w.seq) * q_len + qi;
                    args.part_lse[pslot * kHeads + m] = l_sum > 0.f ? m_used + __log2f(l_sum) : -CUDART_INF_F;
                }
                m_used = -CUDART_INF_F;
                l_part = 0.f;
            }
        }
        if (!ok) *abort_flag = 1;
    } else if (rank == 1 && warp == 1) {
        // ======================================================== accumulator: O issuer (whole warp waits, lane 0 issues)
        // O += P(g) . latent(g) (N = 512 as two MMAs of N = 256 per K step,
        // P from the slot, the latent MN-major from the stage); the first tile
        // of a piece overwrites O after the previous piece's epilogue read it.
        constexpr uint32_t idO = idesc_bf16_f32(kHeads, 256, false, true);
        const uint64_t dP = smem_desc(base + kOffPSlots, 16, 512, kSw64);            // P key halves, K-major
        const uint64_t dV = smem_desc(base + kOffVStages, kChunk, 1024, kSw128);     // latent, MN-major
        TileWalk wo;
        wo.init(args.plan, grp);
        int T_o = wo.valid ? args.seqlens[wo.seq] : 0;
        bool ok = true;
        for (int g = 0; wo.valid && ok && !*abort_flag; ++g) {
            const int slot = g % kPSlots, st = g % kVStages;
            const uint32_t ph = (g / kPSlots) & 1;
            if (!MLA_TW(kTwPFull, warp_wait_cluster(bar(kBarPFull0 + slot), ph, lim))) { ok = false; break; }
            if (!MLA_TW(kTwPFull, warp_wait(bar(kBarRescaled0 + slot), ph, lim))) { ok = false; break; }
            if (!MLA_TW(kTwFull, warp_wait(bar(kBarVFull0 + st), (g / kVStages) & 1, lim))) { ok = false; break; }
            if (wo.first() && wo.seg > 0 &&
                !MLA_TW(kTwOFree, warp_wait(bar(kBarOFree), (wo.seg - 1) & 1, lim))) { ok = false; break; }
            const uint32_t tile = base + kOffVStages + st * kVStageBytes;
            const int valid = T_o - wo.t * kNk;
            if (valid < kNk) zero_rows(tile, 8, valid < 0 ? 0 : valid, lane);
            __syncwarp();
            tc_fence_after();
            if (lane == 0) {
                MLA_TRACE_POINT(15, g);
                const bool first = wo.first();
                const uint64_t a0 = dP + ((slot * kPSlotBytes) >> 4);
                const uint64_t b0 = dV + ((st * kVStageBytes) >> 4);
#pragma unroll
                for (int k = 0; k < 4; ++k)
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf)
                        mma_f16_ss(tmem + kTmemO + 256 * hf, a0 + ((kPHalf * (k >> 1) + 32 * (k & 1)) >> 4),
                                   b0 + ((4 * kChunk * hf + 2048 * k) >> 4), idO, (!first || k > 0) ? 1u : 0u);
                mma_commit(bar(kBarPDone0 + slot));
                mma_commit(bar(kBarVEmpty0 + st));
                if (wo.last()) mma_commit(bar(kBarOFull));
                MLA_TRACE_POINT(2, g);
            }
            __syncwarp();
            const int seq_before = wo.seq;
            wo.advance();
            if (wo.valid && wo.seq != seq_before) T_o = args.seqlens[wo.seq];
        }
        if (!ok) *abort_flag = 1;
    } else if (rank == 1 && warp == 10) {
        // ======================================================== accumulator: slot forwarder (lane 0)
        // Arms each P slot for the scorer's next tile in it (expected bytes),
        // then tells the scorer the slot is free, once the O MMA that read it
        // has completed.
        TileWalk w;
        w.init(args.plan, grp);
        int n_tiles = 0;
        for (TileWalk c = w; c.valid; c.advance()) ++n_tiles;
        const uint32_t slotfree_peer = mapa(bar(kBarSlotFree0), peer);
        bool ok = true;
        if (lane == 0)
            for (int s = 0; s < kPSlots && s < n_tiles; ++s) mbar_arrive_expect_tx(bar(kBarPFull0 + s), kPSlotBytes);
        for (int g = 0; g + kPSlots < n_tiles && ok && !*abort_flag; ++g) {
            const int slot = g % kPSlots;
            if (!warp_wait(bar(kBarPDone0 + slot), (g / kPSlots) & 1, lim)) { ok = false; break; }
            if (lane == 0) {
                mbar_arrive_expect_tx(bar(kBarPFull0 + slot), kPSlotBytes);  // for tile g + kPSlots
                mbar_arrive_remote_relaxed(slotfree_peer + 8 * slot);
            }
        }
        if (!ok) *abort_flag = 1;
    } else if (rank == 1 && softmax_warp) {
        // ======================================================== accumulator: rescale / epilogue warps
        // Two warps per TMEM quarter: half kh owns O columns 256kh..256kh+255
        // of its rows.  Per tile: apply the scorer's rescale factor to O rows
        // whose maximum grew (the whole warp, factor 1 on the other rows),
        // then release the O MMA; at the end of a piece, normalise O and store
        // o_lat (bf16) or the split partial (fp32).
        const float* slots = reinterpret_cast<const float*>(base_ptr + kOffPSlots);
        bool ok = true;
        TileWalk w;
        w.init(args.plan, grp);
        for (int g = 0; w.valid && ok && !*abort_flag; ++g, w.advance()) {
            const int slot = g % kPSlots;
            if (!MLA_TW(kTwXFull, warp_wait_cluster(bar(kBarPFull0 + slot), (g / kPSlots) & 1, lim))) { ok = false; break; }
            // the row data {f, this half's sum of p} of both key halves: read
            // before the slot is released (the scorer refills it once O(g) has
            // completed)
            const float* rowdat = slots + (slot * kPSlotBytes + kPData) / 4 + 2 * m;
            const float f = rowdat[0];
            const float l_sum = rowdat[1] + rowdat[1024 / 4 + 1];
            const bool first = w.first();
            if (!first && __any_sync(0xffffffffu, f != 1.0f)) {
                // O must hold everything up to tile g-1 before it is rescaled
                const int ps = (g - 1) % kPSlots;
                if (!warp_wait(bar(kBarPDone0 + ps), ((g - 1) / kPSlots) & 1, lim)) { ok = false; break; }
                tc_fence_after();
#pragma unroll 1
                for (int c0 = 0; c0 < 256; c0 += 32) {
                    uint32_t v[32];
                    tmem_ld32(tmem + lane_addr + kTmemO + 256 * kh + c0, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * f);
                    tmem_st32(tmem + lane_addr + kTmemO + 256 * kh + c0, v);
                }
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kBarRescaled0 + slot));
            if (threadIdx.x == 64) MLA_TRACE_POINT(5, g);
            if (!w.last()) continue;
            // ---- epilogue: this thread owns O row m, columns 256kh..256kh+255
            if (!warp_wait(bar(kBarOFull), w.seg & 1, lim)) { ok = false; break; }
            tc_fence_after();
            const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
            const int u = w.seq * q_len + qi;
            const int col0 = 256 * kh;
            if (w.whole) {
                __nv_bfloat16* dst = args.o_lat + ((size_t)u * kHeads + m) * kLat + col0;
#pragma unroll 1
                for (int c0 = 0; c0 < 256; c0 += 32) {
                    uint32_t v[32];
                    tmem_ld32(tmem + lane_addr + kTmemO + col0 + c0, v);
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
                const size_t pslot = (size_t)(grp + w.seq) * q_len + qi;
                float* dst = args.part_o + (pslot * (kLat / 8) * kHeads + m) * 8;
#pragma unroll 1
                for (int c0 = 0; c0 < 256; c0 += 32) {
                    uint32_t v[32];
                    tmem_ld32(tmem + lane_addr + kTmemO + col0 + c0, v);
                    tmem_wait_ld();
                    const int o0 = (col0 + c0) / 8;
#pragma unroll
                    for (int j = 0; j < 32; j += 8) {
                        uint32_t o[8];
#pragma unroll
                        for (int q = 0; q < 8; ++q) o[q] = __float_as_uint(__uint_as_float(v[j + q]) * inv);
                        st_global_v8(dst + (size_t)(o0 + j / 8) * kHeads * 8, o[0], o[1], o[2], o[3], o[4], o[5], o[6],
                                     o[7]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kBarOFree));
            if (threadIdx.x == 64) MLA_TRACE_POINT(7, g);
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
    // ---- teardown: nothing this CTA issued may still be running when it exits.
    // On normal completion every stage load, MMA and incoming P slot was
    // waited for by its consumer.  After an expired wait the roles stopped
    // early, so what they had issued is drained here (each wait again bounded).
    __syncthreads();  // every role has stopped issuing; the abort flag is final
    const bool aborted = *abort_flag != 0;
    if (aborted && active && warp == 0 && lane == 0) {  // stage loads in flight
        const int nst = rank == 0 ? kSStages : kVStages;
        const int full0 = rank == 0 ? kBarFull0 : kBarVFull0;
        for (int n = n_loads > nst ? n_loads - nst : 0; n < n_loads; ++n)
            mbar_wait(bar(full0 + n % nst), (n / nst) & 1, lim);
    }
    // Every MMA of the issuer (a commit tracks all prior MMAs of its thread).
    if (warp == 1 && lane == 0) mma_commit(bar(kBarDrain));
    if (warp == 1) mbar_wait(bar(kBarDrain), 0, lim);
    if (aborted && threadIdx.x == 0) atomicOr(args.status, MLA_STATUS_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, kTmemCols);
    if (threadIdx.x == 0) MLA_TRACE_POINT(6, kTraceProlog);
    // The peer may still arrive on this CTA's barriers: neither CTA leaves
    // before both have stopped.  P rows the scorer stored into the
    // accumulator's shared memory with st.async are not ordered by the
    // cluster barrier; they have all landed unless a CTA stopped early, in
    // which case both give them time to land before the shared memory is
    // released.
    cluster_sync();
    const bool peer_aborted = ld_shared_cluster_u32(mapa(abort_addr, peer)) != 0;
    cluster_sync();
    if (aborted || peer_aborted) spin_ns(20000);
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
