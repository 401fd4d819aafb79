// mla_decode.cu -- absorbed-form MLA decode for B200 (sm_100a).
//
// Three kernels behind the C ABI of include/mla_decode.h:
//
//   mla_metadata_kernel  split-KV schedule: the 128-token tiles of all
//                        sequences are laid end to end and cut into equal
//                        contiguous ranges, one per CTA group.
//   mla_decode_kernel    one persistent CTA per SM.  Per 128-token tile:
//                          TMA gathers the tile's two pages through the page
//                          table into a ring of shared-memory slots of one
//                          or two 16 KB chunks (a chunk = 64 columns of the
//                          128 rows, 128-byte swizzled);
//                          S^T = K Q^T on the tensor core (M = 128 tokens,
//                          N = heads x query positions, K = 576) into TMEM;
//                          a column-wise online softmax of S^T (running max
//                          and sum in fp32) writes P^T (bf16);
//                          O^T += V^T P^T (M = 4 x 128 latent dims, K = 128
//                          tokens) accumulates in TMEM over the whole range.
//                        This is the transposed flow of the FlashMLA-ETAP
//                        explainer (gist.science), technical summary,
//                        "Methodology / core mechanism": the long KV length
//                        is the MMA M dimension, the few query columns are N.
//                        Its producer / consumer warp specialisation follows
//                        that page's "Implementation details / pipeline
//                        structure", re-drawn for tcgen05.
//   mla_combine_kernel   merges the fp32 partials of sequences cut into
//                        several pieces through their log-sum-exp (the online
//                        softmax of "FlashMLA: compressing the KV cache",
//                        jsqmd.com, "compute flow" step 4, across CTAs).
//
// The V part of each tile is copied, transposed, from its shared-memory slots
// into a ring of V^T blocks in TMEM by four transposer warps as soon as it
// lands (ldmatrix.trans -> tcgen05.st), and the output MMA reads A = V^T from
// TMEM.  A slot is released once the score MMA and the transposer have read
// it, so the slot ring never waits on the softmax, and a V^T block is released
// as soon as its output MMAs complete.  Warps: producer, score MMA, 4 softmax,
// 4 transposer, output MMA.
//
// The FP8 instances (an e4m3 cache with one fp32 scale per token) feed the
// codes to the tensor cores as they land (kind::f8f6f4): the score MMA reads
// each 128-column unit K-major against q written as two e4m3 terms, the
// softmax writes its weights as two e4m3 terms, and the output MMA reads V^T
// MN-major from a second copy of the latent units that one of the transposer
// warps loads into a V ring (the other three are idle there).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <climits>
#include <cstdlib>
#include <atomic>
#include <mutex>

#include "../../include/mla_decode.h"
#include "sm100_ptx.cuh"

namespace mla {

constexpr int kDQK = MLA_D_QK;
constexpr int kDV = MLA_D_V;
constexpr int kPage = MLA_PAGE;
constexpr int kTile = MLA_TILE;
constexpr int kChunks = kDQK / 64;              // 9 column chunks per row
constexpr uint32_t kChunkBytes = 16384;         // one 64-column chunk of a tile: 128 rows x 128 B
constexpr uint32_t kPageChunkBytes = 8192;      // 64 rows x 128 B
constexpr int kThreads = 352;                   // producer, score MMA, 4 softmax, 4 transposer, output MMA
constexpr int kMaxRing = 16;
constexpr int kMinRingChunks = 4;               // the transposer may hold two chunks while the third lands
constexpr int kMaxBatch = 4096;
constexpr int kMaxSms = 4096;
constexpr int kSchedHeader = 16;
constexpr int kSchedEntry = 8;
constexpr int kSchedMagic = 0x4D4C4144;         // "MLAD"
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // bounded device waits: 2 s
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kTau = 32.f;                    // log2-domain headroom before the reference max moves
constexpr int kMaxVt = 6;                       // V^T blocks TMEM can hold beside O^T and S^T

// Barrier indices inside the "misc" shared-memory region.
constexpr int kBarFull = 0;                        // [kMaxRing] slot loaded
constexpr int kBarEmpty = kMaxRing;                // [kMaxRing] slot read by the score MMA and the transposer
constexpr int kBarQFull = 2 * kMaxRing;
constexpr int kBarQEmpty = kBarQFull + 1;
constexpr int kBarSFull = kBarQEmpty + 1;          // [2] S^T buffer written
constexpr int kBarSEmpty = kBarSFull + 2;          // [2] S^T buffer read into registers
constexpr int kBarPFull = kBarSEmpty + 2;          // [2] P^T buffer written
constexpr int kBarPEmpty = kBarPFull + 2;          // [2] output MMA of that P^T complete
constexpr int kBarVtFull = kBarPEmpty + 2;         // [kMaxVt] V^T block written
constexpr int kBarVtEmpty = kBarVtFull + kMaxVt;   // [kMaxVt] output MMA of that V^T block complete
constexpr int kBarDrain = kBarVtEmpty + kMaxVt;
constexpr int kBarDrainO = kBarDrain + 1;
// FP8 cache (16 or 32 query columns).  The tensor cores read the e4m3 codes
// as they lie in the cache (tcgen05.mma kind::f8f6f4): the ring's slots are
// 16 KB "units", one 128-column group of a tile (128 rows x 128 bytes of
// codes, both pages, 128-byte swizzled), five per tile, the last holding the
// 64 rope columns and the zero fill of its TMA box.  The score MMA reads a
// unit K-major (rows = tokens) and frees it.  A second producer loads the
// tile's four latent units again -- from L2, just read -- into a V ring of
// f8_vring() units after the unit ring, where the output MMA reads them
// MN-major (rows = tokens, the 128 latent dims contiguous) as V^T.  The
// tile's 128 token scales land with its first unit in a ring of 512-byte
// buffers after the V ring.
constexpr int kF8Units = 5;                // per tile: latent columns 0-511 in 4 groups, then the rope group
constexpr uint32_t kF8Half = 8192;         // one page's 64 rows x 128 B of codes
constexpr uint32_t kF8UnitBytes = 16384;   // one ring slot: a unit's codes
template <int N>
__host__ __device__ constexpr int f8_vring()  // V-ring units: one tile's four (the rest of the memory goes to the unit ring)
{
    return 4;
}
// Token scales of tile T are replaced by tile T + 8's once the slot of unit
// 5 (T + 8) - R is free: for R <= 16 a unit of tile T + 4 or later, freed by
// the score MMA of that tile, which waits for the softmax of tile T + 2 to
// have read its S^T buffer -- after the softmax of tile T read the scales.
constexpr int kRawScBufs = 8;
constexpr uint32_t kRawScBytes = kRawScBufs * 512;
// q split into two e4m3 terms per element (see softmax_warps): per unit a hi
// and a lo tile of N rows x 128 B each, stacked, 128-byte swizzled, K-major
// (Cfg::QS8_UNIT, Cfg::QS8).  The bf16 q is loaded into the same bytes and
// split in place.
// FP8 weights: the reference max sits kLift8 below the largest log2 weight
// seen when it last moved, so weights reach 2^kLift8 and stay above e4m3's
// subnormal range (2^-6) down to 2^-13 of the largest; it moves again when a
// weight would pass 2^kTau8 = 430 (e4m3 holds up to 448 = 2^8.81; each move
// rescales O^T after waiting for the previous tile's output MMA, and 2^8.75
// rather than 2^8 made that 1.5 us per call rarer on both FP8 workloads).  l
// and lse use the same reference, so the result does not depend on it.
constexpr float kLift8 = 7.f;
constexpr float kTau8 = 8.75f;
// The barrier block below keeps the layout of an earlier design (the bf16
// instances are laid out exactly as before); the FP8 instance uses its first
// entry for "q split written".
constexpr int kBarF8Full = kBarDrainO + 1;
constexpr int kBarQsFull = kBarF8Full;
constexpr int kBarVFull = kBarF8Full + 1;          // [f8_vring] a V-ring unit landed
constexpr int kBarVEmpty = kBarF8Full + 8;         // [f8_vring] the output MMA has read it
constexpr int kScBufs = 4;
constexpr uint32_t kScBytes = kScBufs * 128 * 4;   // (unused; kept for the layout of the bf16 instances)
constexpr uint32_t kQScaleBytes = 128;              // FP8: the per-row q scales
constexpr int kBarF8Reserved = kBarF8Full + 8 + 2 * kScBufs;
static_assert(kBarVFull + 5 <= kBarVEmpty && kBarVEmpty + 5 <= kBarF8Reserved, "FP8 V-ring barriers");
constexpr int kNumBars = kBarF8Reserved;
// The reduction buffers after the barriers are read as float4: keep them
// 16-byte aligned (rounded to 128 B).
constexpr uint32_t kMiscRedOffset = (kNumBars * 8 + 127) / 128 * 128;
static_assert(kMiscRedOffset % 16 == 0, "reduction buffers must be 16-byte aligned");

template <int N>
__host__ __device__ constexpr uint32_t misc_bytes()
{
    // barriers, max-reduction buffer [4][N], sum buffer [4][N], reference max [N], shift [N],
    // tmem holder, abort flag, 2 spare words, transposer scratch [128]
    return kMiscRedOffset + (4 * N + 4 * N + N + N) * 4 + 16 + 128 * 4;
}

struct DecodeParams {
    const int32_t *block_table;
    const int32_t *seqlens;
    const int32_t *sched;
    const int32_t *split_base;
    float *ws_o;
    float *ws_lse;
    uint16_t *out;
    float *lse;
    int32_t *err;
    int B, s_q, H, G, num_sms, num_tuples, max_blocks, ring;
    int max_pieces;  // workspace capacity in (piece, group) slots
    int64_t num_blocks;
    float scale_log2;
    int debug_stall_cta;  // test hook: this CTA never loads its first chunk (-1: none)
};

struct Range {
    int b0, t0, b1, t1, split0;
};

__device__ __forceinline__ int tiles_of(int L) { return L > 0 ? (L + kTile - 1) / kTile : 0; }

__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                             int32_t *err, bool honour_abort = true)
{
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = ptx::globaltimer_ns();
    uint32_t spins = 0;
    while (true) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if ((++spins & 3u) == 0) {
            if (honour_abort && *abort_flag) return false;
            if (ptx::globaltimer_ns() - t0 > kWaitLimitNs) {
                *abort_flag = 1;
                atomicOr(err, MLA_DEVERR_TIMEOUT);
                return false;
            }
        }
    }
}

__device__ __forceinline__ float warp_max(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

__device__ __forceinline__ float warp_sum(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// ============================================================== metadata
// One block.  prefix[b] = tiles of sequences < b; a CTA group k owns the
// flattened tiles [k * per, min((k + 1) * per, total)).  Sequence b is cut
// into one piece per group whose range meets it; those pieces are numbered
// from split_base[b].
constexpr int kMetaThreads = 128;

__device__ int block_exclusive_scan(int *arr, int n, int *warp_sums)
{
    // arr[0..n) -> exclusive prefix in place; returns the total.
    const int tid = threadIdx.x;
    const int per = (n + kMetaThreads - 1) / kMetaThreads;
    const int lo = min(n, tid * per), hi = min(n, lo + per);
    int local = 0;
    for (int k = lo; k < hi; ++k) local += arr[k];
    // inclusive scan of `local` over the block
    const int lane = tid & 31, warp = tid >> 5;
    int x = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < kMetaThreads / 32 ? warp_sums[lane] : 0;  // lanes past the last warp add nothing
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        warp_sums[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    int run = x - local + (warp > 0 ? warp_sums[warp - 1] : 0);
    const int total = warp_sums[31];
    for (int k = lo; k < hi; ++k) {
        const int v = arr[k];
        arr[k] = run;
        run += v;
    }
    __syncthreads();
    return total;
}

// Largest b in [0, B) with prefix[b] <= x (prefix non-decreasing, prefix[0] = 0).
__device__ int last_at_or_below(const int *prefix, int B, int x)
{
    int lo = 0, hi = B - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (prefix[mid] <= x) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Header and error word of the schedule (thread 0).
__device__ __forceinline__ void write_sched_header(int32_t *sched, int bad, int B, int s_q, int H, int num_sms,
                                                   int num_tuples, int G, int per, int total, int total_splits)
{
    sched[0] = bad ? MLA_DEVERR_SEQLEN : 0;
    sched[1] = kSchedMagic;
    sched[2] = B;
    sched[3] = s_q;
    sched[4] = H;
    sched[5] = num_sms;
    sched[6] = num_tuples;
    sched[7] = G;
    sched[8] = per;
    sched[9] = total;
    sched[10] = total_splits;
    for (int k = 11; k < kSchedHeader; ++k) sched[k] = 0;
}

// Work range of CTA group k: {b0, first tile in b0, b1, end tile in b1,
// piece index within b0}, or {-1, 0, -1, 0, 0} past the last tile.
__device__ __forceinline__ void write_sched_entry(int32_t *sched, int k, int per, int total, int b0, int pre_b0,
                                                  int b1, int pre_b1)
{
    int32_t *e = sched + kSchedHeader + k * kSchedEntry;
    const int start = k * per;
    if (start >= total) {
        e[0] = -1; e[1] = 0; e[2] = -1; e[3] = 0; e[4] = 0; e[5] = 0; e[6] = 0; e[7] = 0;
        return;
    }
    const int end = min(start + per, total);
    e[0] = b0;
    e[1] = start - pre_b0;
    e[2] = b1;
    e[3] = end - pre_b1;
    e[4] = k - pre_b0 / per;  // index of this group's piece of sequence b0
    e[5] = 0; e[6] = 0; e[7] = 0;
}

// Batches of at most 32 sequences: one warp, prefix sums by shuffles, no
// block barrier.  Lane b holds sequence b.
__device__ void metadata_warp(const int32_t *__restrict__ seqlens, int B, int s_q, int H, int num_sms,
                              int num_tuples, int G, int32_t *__restrict__ sched, int32_t *__restrict__ split_base,
                              int *pre_s)
{
    const int lane = threadIdx.x;
    int L = lane < B ? seqlens[lane] : 0;
    const bool bad = __any_sync(0xffffffffu, L < 0);
    L = max(L, 0);
    const int nt = tiles_of(L);
    int inc = nt;  // inclusive prefix of tiles
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
    }
    const int pre = inc - nt;  // exclusive prefix: first tile of sequence `lane`
    const int total = __shfl_sync(0xffffffffu, inc, 31);
    const int per = total > 0 ? (total + num_tuples - 1) / num_tuples : 1;
    pre_s[lane] = pre;
    __syncwarp();
    for (int k = lane; k < num_tuples; k += 32) {
        const int start = k * per;
        if (start >= total) {
            write_sched_entry(sched, k, per, total, 0, 0, 0, 0);
            continue;
        }
        const int end = min(start + per, total);
        const int b0 = last_at_or_below(pre_s, B, start);
        const int b1 = last_at_or_below(pre_s, B, end - 1);
        write_sched_entry(sched, k, per, total, b0, pre_s[b0], b1, pre_s[b1]);
    }
    const int ns = nt > 0 ? (pre + nt - 1) / per - pre / per + 1 : 0;
    int ninc = ns;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, ninc, o);
        if (lane >= o) ninc += y;
    }
    if (lane < B) split_base[lane] = ninc - ns;
    const int total_splits = __shfl_sync(0xffffffffu, ninc, 31);
    if (lane == 0) {
        split_base[B] = total_splits;
        write_sched_header(sched, bad, B, s_q, H, num_sms, num_tuples, G, per, total, total_splits);
    }
}

// The schedule in shared memory sized to the batch (2 (B + 1) + 33 ints,
// dynamic), so that for small batches the block fits on an SM beside an
// attention CTA and every attention CTA can start at once.
__global__ void __launch_bounds__(kMetaThreads, 1)
mla_metadata_kernel(const int32_t *__restrict__ seqlens, int B, int s_q, int H, int num_sms,
                    int num_tuples, int G, int32_t *__restrict__ sched, int32_t *__restrict__ split_base)
{
    // The attention grid may become resident now: it runs its prologue and
    // then waits for this grid to complete before reading the schedule.
    ptx::griddep_launch_dependents();
    extern __shared__ uint8_t smem_raw[];
    if (B <= 32) {
        if (threadIdx.x < 32)
            metadata_warp(seqlens, B, s_q, H, num_sms, num_tuples, G, sched, split_base,
                          reinterpret_cast<int *>(smem_raw));
        return;
    }
    int *prefix = reinterpret_cast<int *>(smem_raw);  // [B + 1]
    int *nsplit = prefix + (B + 1);   // [B + 1]
    int *warp_sums = nsplit + (B + 1);  // [32]
    int &bad_len = warp_sums[32];
    const int tid = threadIdx.x;
    if (tid == 0) bad_len = 0;
    __syncthreads();
    for (int b = tid; b < B; b += kMetaThreads) {
        int L = seqlens[b];
        if (L < 0) {
            bad_len = 1;
            L = 0;
        }
        prefix[b] = tiles_of(L);
    }
    __syncthreads();
    const int total = block_exclusive_scan(prefix, B, warp_sums);
    if (tid == 0) prefix[B] = total;
    __syncthreads();
    const int per = total > 0 ? (total + num_tuples - 1) / num_tuples : 1;

    for (int k = tid; k < num_tuples; k += kMetaThreads) {
        const int start = k * per;
        if (start >= total) {
            write_sched_entry(sched, k, per, total, 0, 0, 0, 0);
            continue;
        }
        const int end = min(start + per, total);
        const int b0 = last_at_or_below(prefix, B, start);
        const int b1 = last_at_or_below(prefix, B, end - 1);
        write_sched_entry(sched, k, per, total, b0, prefix[b0], b1, prefix[b1]);
    }
    for (int b = tid; b < B; b += kMetaThreads) {
        const int nt = prefix[b + 1] - prefix[b];
        nsplit[b] = nt > 0 ? (prefix[b + 1] - 1) / per - prefix[b] / per + 1 : 0;
    }
    __syncthreads();
    const int total_splits = block_exclusive_scan(nsplit, B, warp_sums);
    for (int b = tid; b < B; b += kMetaThreads) split_base[b] = nsplit[b];
    if (tid == 0) {
        split_base[B] = total_splits;
        write_sched_header(sched, bad_len, B, s_q, H, num_sms, num_tuples, G, per, total, total_splits);
    }
}

// All lanes of the calling warp wait; the outcome is agreed warp-wide so the
// warp stays converged even when a bounded wait runs out in some lanes only.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag, int32_t *err,
                                          bool honour_abort = true)
{
    const bool ok = wait_bounded(bar, parity, abort_flag, err, honour_abort);
    return __all_sync(0xffffffffu, ok);
}

// Page-table window of 32 pages.  table_entry loads lane j's entry for page
// `first + j` whenever it lies inside the table row, so the load need not
// wait for the length; checked_page then gives the physical block (0 for
// pages outside [0, npages), and, with an error bit, for entries that do not
// name a block of the cache).
__device__ __forceinline__ int table_entry(const int32_t *bt, int first, const DecodeParams &p, int lane)
{
    const int idx = first + lane;
    return (idx >= 0 && idx < p.max_blocks) ? __ldg(bt + idx) : 0;
}

__device__ __forceinline__ int checked_page(int raw, int first, int npages, const DecodeParams &p, int lane)
{
    const int idx = first + lane;
    int id = 0;
    if (idx < npages) {
        if (idx >= p.max_blocks) {
            atomicOr(p.err, MLA_DEVERR_SEQLEN);
        } else if (raw < 0 || static_cast<int64_t>(raw) >= p.num_blocks) {
            atomicOr(p.err, MLA_DEVERR_BLOCK_TABLE);
        } else {
            id = raw;
        }
    }
    return id;
}

__device__ __forceinline__ int load_pages(const int32_t *bt, int first, int npages, const DecodeParams &p, int lane)
{
    return checked_page(table_entry(bt, first, p, lane), first, npages, p, lane);
}

// ================================================================ decode
// Per-shape constants.  TMEM (512 columns of 128 lanes x 32 bit) holds, left
// to right: O^T as 4 blocks of N columns (latent dims 128j..128j+127 on the
// lanes), NS buffers of S^T (N columns each), and a ring of NVT V^T blocks of
// 64 columns (128 tokens as bf16 pairs; latent dims on the lanes).
template <int N, int SQ>
struct Cfg {
    static constexpr int HG = N / SQ;                      // heads per CTA
    static constexpr int NCH = N / 16;                     // 16-column TMEM chunks
    static constexpr int NS = N <= 32 ? 2 : 1;             // S^T buffers
    static constexpr uint32_t QCHUNK = N * 128u;           // bytes: 64 columns of N rows
    static constexpr uint32_t QBYTES = kChunks * QCHUNK;   // N x 576 bf16
    static constexpr uint32_t PBYTES = 2 * 2 * QCHUNK;     // 2 P^T buffers of N x 128 bf16
    static constexpr uint32_t S_COL = 4 * N;
    // FP8 instance: each MMA has 2N columns, n and N + n holding the hi and
    // lo terms of column n; O^T blocks are 2N wide, S^T from column 8N.
    static constexpr uint32_t S_COL8 = 8 * N;
    static constexpr uint32_t QS8_UNIT = 2 * N * 128u;        // FP8: one unit of q's stacked e4m3 terms
    static constexpr uint32_t QS8 = kF8Units * QS8_UNIT;       // holds the bf16 q too (9 x 128 N bytes)
    static constexpr uint32_t VT_COL = (S_COL + NS * N + 63) / 64 * 64;
    static constexpr int NVT = (512 - static_cast<int>(VT_COL)) / 64;
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(NVT >= 3 && NVT <= kMaxVt, "V^T ring does not fit");
    // Chunks per ring slot.  One slot is one barrier pair and one producer
    // round; the loads of a slot (two 8 KB boxes per chunk) are issued back to
    // back.  Measured on the 16-column shape, 2-chunk slots stream the cache
    // faster than 1-chunk slots (1.5 us of 108 at a 64K context); at 32
    // columns they made no difference, and at 64 columns, whose ring is the
    // smallest, rounding the ring down to whole 2- or 3-chunk slots cost 30
    // and 60 us.
    static constexpr int CPS = N == 16 ? 2 : 1;
    static constexpr int SPT = (kChunks + CPS - 1) / CPS;   // slot uses per tile
    static constexpr uint32_t SLOT_BYTES = CPS * kChunkBytes;
    // Arrivals that free a slot: the score MMA's commit and two transposer
    // warps per latent chunk; the score MMA stands in for the transposer on
    // the rope chunk (and on the unused chunk positions of the last slot).
    static constexpr int EMPTY_ARRIVALS = 1 + 2 * CPS;
    static constexpr int LAST_SLOT_COMMITS = 1 + 2 * (CPS - (kChunks - 1 - (SPT - 1) * CPS));
    static_assert(CPS >= 1 && CPS <= 3, "chunks per slot");
};

struct Smem {
    uint32_t ring, q, p;     // shared-window addresses: slot ring, Q, P^T buffers
    uint32_t slot_bytes;     // bytes per ring slot
    uint32_t f8;             // shared-window address of the FP8 token-scale buffers (FP8 cache only)
    float *tscale;           // FP8: the per-row q scales 2^-a_n [N]
    uint32_t bars;           // address of barrier 0
    float *red, *lred;       // column-max exchange [4][N], sum exchange [4][N]
    float *mu, *shift;       // reference max [N], its last shift [N]
    uint32_t scratch;        // shared-window address of 128 words for the transposer's load fences
    uint32_t *tmem_holder;
    volatile int *abort_flag;
    __device__ __forceinline__ uint32_t bar(int i) const { return bars + 8u * i; }
    __device__ __forceinline__ uint32_t slot(int s) const { return ring + slot_bytes * s; }
};

// Output of one range: the column sums of the four softmax warps are reduced,
// O^T is normalised and written either as the final out/lse or as the fp32
// piece for the combine kernel.  O^T must be complete (and fenced) when this
// is called.  `l` holds the calling thread's partial sums in the fragment
// layout of softmax_warps.
template <int N, int SQ, bool F8 = false>
__device__ void range_epilogue(const DecodeParams &p, const Smem &sm, uint32_t tmem, int b, int split, int g,
                               const float (&l)[N / 8][2])
{
    using C = Cfg<N, SQ>;
    constexpr int HG = C::HG;
    constexpr int NG = N / 8;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const int tid = threadIdx.x - 64;
    const int c2 = 2 * (lane & 3);
    const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
#pragma unroll
    for (int gi = 0; gi < NG; ++gi)
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
            float s = l[gi][jj];
            s += __shfl_xor_sync(0xffffffffu, s, 4);
            s += __shfl_xor_sync(0xffffffffu, s, 8);
            s += __shfl_xor_sync(0xffffffffu, s, 16);
            if ((lane >> 2) == 0) sm.lred[wq * N + 8 * gi + c2 + jj] = s;
        }
    __syncwarp();
    ptx::named_bar_sync(1, 128);
    // Thread n < N totals column n once: its reciprocal goes to sm.shift (free
    // between ranges) for every thread, its lse is written below.
    float ln_own = 0.f;
    if (tid < N) {
        ln_own = (sm.lred[tid] + sm.lred[N + tid]) + (sm.lred[2 * N + tid] + sm.lred[3 * N + tid]);
        sm.shift[tid] = ln_own > 0.f ? 1.f / ln_own : 0.f;
    }
    ptx::named_bar_sync(1, 128);
    float linv[N];
#pragma unroll
    for (int n4 = 0; n4 < N / 4; ++n4) {
        const float4 a = reinterpret_cast<const float4 *>(sm.shift)[n4];
        linv[4 * n4 + 0] = a.x;
        linv[4 * n4 + 1] = a.y;
        linv[4 * n4 + 2] = a.z;
        linv[4 * n4 + 3] = a.w;
    }

    const int nsplit = p.split_base[b + 1] - p.split_base[b];
    const bool final_out = nsplit <= 1;
    int piece = (p.split_base[b] + split) * p.G + g;
    bool write_ok = true;
    if (!final_out && (piece < 0 || piece >= p.max_pieces)) {
        if (tid == 0) atomicOr(p.err, MLA_DEVERR_SCHEDULE);
        write_ok = false;
        piece = 0;
    }
    // Row n = i HG + hl of the piece is (piece N + n) 512 floats in; of the
    // final output, ((b SQ + i) H + g HG + hl) 512 bf16.  With the bases and
    // the per-position stride in registers, each element is one multiply and
    // one store at a constant offset; up to 32 columns are loaded from TMEM
    // per wait.  (A range switch at 64 columns spent ~12 us here when every
    // element recomputed its 64-bit address and each 16 columns waited.)
    constexpr int CW = N < 32 ? N : 32;
    float *const wbase = p.ws_o + static_cast<int64_t>(piece) * N * kDV;
    uint16_t *const obase = p.out + (static_cast<int64_t>(b) * SQ * p.H + g * HG) * kDV;
    const int64_t ostride = static_cast<int64_t>(p.H) * kDV;  // between query positions
#pragma unroll 1
    for (int j = 0; j < 4; ++j) {
        const int dim = j * 128 + row;
#pragma unroll
        for (int c0 = 0; c0 < N; c0 += CW) {
            float v[CW / 16][16];
            if constexpr (F8) {  // block j is 2N wide: add its hi and lo halves
                float u[CW / 16][16];
#pragma unroll
                for (int k = 0; k < CW / 16; ++k) {
                    ptx::tmem_ld16(tmem + lane_base + j * 2 * N + c0 + 16 * k, v[k]);
                    ptx::tmem_ld16(tmem + lane_base + j * 2 * N + N + c0 + 16 * k, u[k]);
                }
                ptx::tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < CW / 16; ++k)
#pragma unroll
                    for (int e = 0; e < 16; ++e) v[k][e] += u[k][e];
            } else {
#pragma unroll
                for (int k = 0; k < CW / 16; ++k) ptx::tmem_ld16(tmem + lane_base + j * N + c0 + 16 * k, v[k]);
                ptx::tmem_wait_ld();
            }
            if (final_out) {
#pragma unroll
                for (int e = 0; e < CW; ++e) {
                    const int n = c0 + e, i = n / HG, hl = n % HG;
                    obase[i * ostride + hl * kDV + dim] =
                        __bfloat16_as_ushort(__float2bfloat16_rn(v[e / 16][e % 16] * linv[n]));
                }
            } else if (write_ok) {
                float *const wrow = wbase + dim;
#pragma unroll
                for (int e = 0; e < CW; ++e) wrow[(c0 + e) * kDV] = v[e / 16][e % 16] * linv[c0 + e];
            }
        }
    }
    if (tid < N) {
        const int n = tid;
        const int i = n / HG, hl = n % HG;
        const float ln = ln_own;
        const float val = ln > 0.f ? (sm.mu[n] + log2f(ln)) * kLn2 : -INFINITY;
        if (final_out)
            p.lse[(static_cast<int64_t>(b) * SQ + i) * p.H + g * HG + hl] = val;
        else if (write_ok)
            p.ws_lse[(static_cast<int64_t>(piece) * SQ + i) * HG + hl] = val;
    }
    __syncwarp();
    ptx::tc_fence_before();
}

// -- producer warp: Q per range, then each tile's 9 chunks in order --------
template <int N, int SQ, bool F8>
__device__ void producer_warp(const DecodeParams &p, const Range &w, int g, const Smem &sm,
                              const CUtensorMap *kv_map, const CUtensorMap *q_map, const CUtensorMap *sc_map)
{
    using C = Cfg<N, SQ>;
    const int lane = threadIdx.x & 31;
    const uint32_t R = static_cast<uint32_t>(p.ring);
    uint32_t cc = 0;  // ring slot uses so far (FP8 cache: one per unit)
    int qi = 0;       // Q loads so far
    bool ok = true;
    for (int b = w.b0; b <= w.b1 && ok; ++b) {
        const int tb = (b == w.b0) ? w.t0 : 0;
        const int32_t *bt = p.block_table + static_cast<int64_t>(b) * p.max_blocks;
        int win = 2 * tb;
        // The range's first two page-table windows are fetched together with
        // the length rather than after it (one memory round trip less before
        // the first cache load); the entries lie inside the table row, and
        // only those below the page count are used.
        const int raw_cur = table_entry(bt, win, p, lane);
        const int raw_nxt = table_entry(bt, win + 32, p, lane);
        const int L = max(0, __ldg(p.seqlens + b));
        const int nt = tiles_of(L);
        const int te = min((b == w.b1) ? w.t1 : nt, nt);
        if (tb >= te) continue;
        const int npages = (L + kPage - 1) / kPage;
        int cur = checked_page(raw_cur, win, npages, p, lane);
        int nxt = checked_page(raw_nxt, win + 32, npages, p, lane);

        if (!(ok = warp_wait(sm.bar(kBarQEmpty), (qi & 1) ^ 1, sm.abort_flag, p.err))) break;
        ptx::mbar_arrive_expect_tx_elect(sm.bar(kBarQFull), C::QBYTES);
#pragma unroll 1
        for (int i = 0; i < SQ; ++i)
#pragma unroll 1
            for (int c = 0; c < kChunks; ++c)
                ptx::tma_load_2d_elect(sm.q + c * C::QCHUNK + i * C::HG * 128u, q_map, sm.bar(kBarQFull), c * 64,
                                       (b * SQ + i) * p.H + g * C::HG);
        ++qi;

        for (int t = tb; t < te && ok; ++t) {
            if (2 * t >= win + 32) {
                win += 32;
                cur = nxt;
                nxt = load_pages(bt, win + 32, npages, p, lane);
            }
            const int phys0 = __shfl_sync(0xffffffffu, cur, 2 * t - win);
            const int phys1 = __shfl_sync(0xffffffffu, cur, 2 * t + 1 - win);
            const bool live1 = (t * kTile + kPage) < L;
            if constexpr (F8) {
                // FP8: the codes of the tile's five 128-column groups, one ring
                // slot each, the token scales with the first.
                const uint32_t b8 = live1 ? 2 * kF8Half : kF8Half;
                const uint32_t bsc = live1 ? 512u : 256u;
                const uint32_t scb = sm.f8 + ((cc / kF8Units) % kRawScBufs) * 512u;
#pragma unroll 1
                for (int k = 0; k < kF8Units; ++k) {
                    const uint32_t u = cc + k;
                    const int slot = static_cast<int>(u % R);
                    if (!warp_wait(sm.bar(kBarEmpty + slot), ((u / R) & 1) ^ 1, sm.abort_flag, p.err)) {
                        ok = false;
                        cc += k;
                        break;
                    }
                    ptx::mbar_arrive_expect_tx_elect(sm.bar(kBarFull + slot), b8 + (k == 0 ? bsc : 0u));
                    if (u == 0 && static_cast<int>(blockIdx.x) == p.debug_stall_cta) continue;
                    const uint32_t dst = sm.slot(slot);
                    ptx::tma_load_3d_elect(dst, kv_map, sm.bar(kBarFull + slot), 128 * k, 0, phys0);
                    if (live1)
                        ptx::tma_load_3d_elect(dst + kF8Half, kv_map, sm.bar(kBarFull + slot), 128 * k, 0, phys1);
                    if (k == 0) {
                        ptx::tma_load_2d_elect(scb, sc_map, sm.bar(kBarFull + slot), 0, phys0);
                        if (live1) ptx::tma_load_2d_elect(scb + 256, sc_map, sm.bar(kBarFull + slot), 0, phys1);
                    }
                }
                if (ok) cc += kF8Units;
                continue;
            }
            const uint32_t bytes = live1 ? 2 * kPageChunkBytes : kPageChunkBytes;
#pragma unroll 1
            for (int s = 0; s < C::SPT; ++s) {
                const uint32_t u = cc + s;
                const int slot = static_cast<int>(u % R);
                if (!warp_wait(sm.bar(kBarEmpty + slot), ((u / R) & 1) ^ 1, sm.abort_flag, p.err)) {
                    ok = false;
                    cc += s;  // uses issued so far in this tile
                    break;
                }
                const int c0 = s * C::CPS, c1 = min(c0 + C::CPS, kChunks);
                ptx::mbar_arrive_expect_tx_elect(sm.bar(kBarFull + slot), bytes * (c1 - c0));
                // Test hook for the bounded waits: the slot is announced but
                // never loaded, so its consumers' waits run out.
                if (u == 0 && static_cast<int>(blockIdx.x) == p.debug_stall_cta) continue;
                const uint32_t dst = sm.slot(slot);
#pragma unroll 1
                for (int c = c0; c < c1; ++c) {
                    const uint32_t d = dst + (c - c0) * kChunkBytes;
                    ptx::tma_load_3d_elect(d, kv_map, sm.bar(kBarFull + slot), c * 64, 0, phys0);
                    if (live1)
                        ptx::tma_load_3d_elect(d + kPageChunkBytes, kv_map, sm.bar(kBarFull + slot), c * 64, 0,
                                               phys1);
                }
            }
            if (ok) cc += C::SPT;
        }
    }
    if (!ok) {
        // Let every load this warp issued land before the CTA exits.
        const uint32_t RR = R;
        const int full0 = kBarFull;
        const uint32_t first = cc > RR ? cc - RR : 0;
        for (uint32_t u = first; u < cc; ++u)
            warp_wait(sm.bar(full0 + static_cast<int>(u % RR)), (u / RR) & 1, sm.abort_flag, p.err, false);
    }
}

// -- score-MMA warp: S^T(t) into S buffer t % NS, chunk by chunk ------------
template <int N, int SQ>
__device__ void score_mma_warp(const DecodeParams &p, const Range &w, const Smem &sm, uint32_t tmem)
{
    using C = Cfg<N, SQ>;
    constexpr uint32_t idS = ptx::idesc_bf16_f32(128, N, false, false);  // K (cache) K-major, Q K-major
    const uint32_t R = static_cast<uint32_t>(p.ring);
    uint32_t cc = 0, it = 0;
    int qi = 0;
    bool ok = true;
    for (int b = w.b0; b <= w.b1 && ok; ++b) {
        const int L = max(0, __ldg(p.seqlens + b));
        const int nt = tiles_of(L);
        const int tb = (b == w.b0) ? w.t0 : 0;
        const int te = min((b == w.b1) ? w.t1 : nt, nt);
        if (tb >= te) continue;
        if (!(ok = warp_wait(sm.bar(kBarQFull), qi & 1, sm.abort_flag, p.err))) break;
        ++qi;
        ptx::tc_fence_after();
        for (int t = tb; t < te && ok; ++t) {
            const uint32_t sb = it % C::NS, su = it / C::NS;
            // the softmax has read the previous S^T of this buffer into registers
            if (su >= 1 && !(ok = warp_wait(sm.bar(kBarSEmpty + sb), (su & 1) ^ 1, sm.abort_flag, p.err))) break;
            ptx::tc_fence_after();
            const uint32_t d = tmem + C::S_COL + sb * N;
#pragma unroll 1
            for (int c = 0; c < kChunks; ++c) {
                const int s = c / C::CPS, cs = c - s * C::CPS;
                const uint32_t u = cc + s;
                const int slot = static_cast<int>(u % R);
                if (cs == 0 && !(ok = warp_wait(sm.bar(kBarFull + slot), (u / R) & 1, sm.abort_flag, p.err))) break;
                ptx::tc_fence_after();
                const uint32_t a0 = sm.slot(slot) + cs * kChunkBytes;
                const uint32_t b0 = sm.q + c * C::QCHUNK;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    ptx::mma_bf16_ss_elect(d, ptx::desc_sw128(a0 + 32u * k, 16, 1024),
                                           ptx::desc_sw128(b0 + 32u * k, 16, 1024), idS, (c | k) != 0);
                // a slot is free after 1 + 2 CPS arrivals: this commit, once
                // its last chunk's MMAs are issued, and one from each of the
                // two transposer warps per latent chunk that read it; the
                // rope chunk is not transposed, so the last slot takes the
                // missing arrivals here
                if (c == kChunks - 1) {
#pragma unroll 1
                    for (int i = 0; i < C::LAST_SLOT_COMMITS; ++i) ptx::mma_commit_elect(sm.bar(kBarEmpty + slot));
                } else if (cs == C::CPS - 1) {
                    ptx::mma_commit_elect(sm.bar(kBarEmpty + slot));
                }
            }
            if (!ok) break;
            ptx::mma_commit_elect(sm.bar(kBarSFull + sb));
            if (t == te - 1) ptx::mma_commit_elect(sm.bar(kBarQEmpty));
            cc += C::SPT;
            ++it;
        }
    }
    ptx::mma_commit_elect(sm.bar(kBarDrain));
    warp_wait(sm.bar(kBarDrain), 0, sm.abort_flag, p.err, false);
}

// -- output-MMA warp: O^T += V^T (TMEM ring) . P^T (shared memory) ----------
// Tile t's four 128-dim blocks are V^T blocks v = 4t .. 4t+3 of the ring; each
// block is handed back to the transposer as soon as its 8 MMAs complete.
template <int N, int SQ>
__device__ void output_mma_warp(const DecodeParams &p, const Range &w, const Smem &sm, uint32_t tmem)
{
    using C = Cfg<N, SQ>;
    constexpr uint32_t idO = ptx::idesc_bf16_f32(128, N, false, false);  // A in TMEM, P^T K-major
    constexpr uint32_t NVT = C::NVT;
    uint32_t it = 0, v = 0;
    bool ok = true;
    for (int b = w.b0; b <= w.b1 && ok; ++b) {
        const int L = max(0, __ldg(p.seqlens + b));
        const int nt = tiles_of(L);
        const int tb = (b == w.b0) ? w.t0 : 0;
        const int te = min((b == w.b1) ? w.t1 : nt, nt);
        for (int t = tb; t < te && ok; ++t) {
            const uint32_t pb = it & 1, pu = it >> 1;
            if (!(ok = warp_wait(sm.bar(kBarPFull + pb), pu & 1, sm.abort_flag, p.err))) break;
            ptx::tc_fence_after();
            const uint32_t pa = sm.p + pb * 2 * C::QCHUNK;
#pragma unroll 1
            for (int j = 0; j < 4; ++j) {
                const uint32_t vb = v % NVT, vu = v / NVT;
                if (!(ok = warp_wait(sm.bar(kBarVtFull + vb), vu & 1, sm.abort_flag, p.err))) break;
                ptx::tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    ptx::mma_bf16_ts_elect(tmem + j * N, tmem + C::VT_COL + 64 * vb + 8 * kk,
                                           ptx::desc_sw128(pa + (kk >> 2) * C::QCHUNK + 32u * (kk & 3), 16, 1024),
                                           idO, (t != tb) || (kk != 0));
                ptx::mma_commit_elect(sm.bar(kBarVtEmpty + vb));
                ++v;
            }
            if (!ok) break;
            ptx::mma_commit_elect(sm.bar(kBarPEmpty + pb));
            ++it;
        }
    }
    ptx::mma_commit_elect(sm.bar(kBarDrainO));
    warp_wait(sm.bar(kBarDrainO), 0, sm.abort_flag, p.err, false);
}

// -- FP8 cache: the two MMA warps on the e4m3 codes ------------------------
// Score MMA: S^T(t) = sum over the tile's five units of K_unit q_unit^T, with
// q as its two e4m3 terms stacked as 2N rows (hi rows 0..N-1, lo rows N..2N-1,
// so S^T has 2N columns whose halves the softmax adds), K = 32 codes per
// instruction.  Every unit's slot is free once its instructions complete (the
// output MMA reads its own copy of the latent units from the V ring).
template <int N, int SQ>
__device__ void score_mma_warp_f8(const DecodeParams &p, const Range &w, const Smem &sm, uint32_t tmem)
{
    using C = Cfg<N, SQ>;
    constexpr uint32_t idS = ptx::idesc_e4m3_f32(128, 2 * N, false, false);  // codes K-major, q terms K-major
    const uint32_t R = static_cast<uint32_t>(p.ring);
    const uint32_t qs = sm.q;
    uint32_t cc = 0, it = 0;
    int qi = 0;
    bool ok = true;
    for (int b = w.b0; b <= w.b1 && ok; ++b) {
        const int L = max(0, __ldg(p.seqlens + b));
        const int nt = tiles_of(L);
        const int tb = (b == w.b0) ? w.t0 : 0;
        const int te = min((b == w.b1) ? w.t1 : nt, nt);
        if (tb >= te) continue;
        if (!(ok = warp_wait(sm.bar(kBarQsFull), qi & 1, sm.abort_flag, p.err))) break;
        ++qi;
        ptx::tc_fence_after();
        for (int t = tb; t < te && ok; ++t) {
            const uint32_t sb = it % C::NS, su = it / C::NS;
            if (su >= 1 && !(ok = warp_wait(sm.bar(kBarSEmpty + sb), (su & 1) ^ 1, sm.abort_flag, p.err))) break;
            ptx::tc_fence_after();
            const uint32_t d = tmem + C::S_COL8 + sb * 2 * N;
#pragma unroll 1
            for (int k = 0; k < kF8Units; ++k) {
                const uint32_t u = cc + k;
                const int slot = static_cast<int>(u % R);
                if (!(ok = warp_wait(sm.bar(kBarFull + slot), (u / R) & 1, sm.abort_flag, p.err))) break;
                ptx::tc_fence_after();
                const uint32_t a0 = sm.slot(slot);
                const uint32_t q0 = qs + k * C::QS8_UNIT;
                const int steps = (k == kF8Units - 1) ? 2 : 4;  // the rope unit: 64 columns
#pragma unroll 1
                for (int kk = 0; kk < steps; ++kk)
                    ptx::mma_e4m3_ss_elect(d, ptx::desc_sw128(a0 + 32u * kk, 16, 1024),
                                           ptx::desc_sw128(q0 + 32u * kk, 16, 1024), idS, (k | kk) != 0);
                ptx::mma_commit_elect(sm.bar(kBarEmpty + slot));
            }
            if (!ok) break;
            ptx::mma_commit_elect(sm.bar(kBarSFull + sb));
            if (t == te - 1) ptx::mma_commit_elect(sm.bar(kBarQEmpty));
            cc += kF8Units;
            ++it;
        }
    }
    ptx::mma_commit_elect(sm.bar(kBarDrain));
    warp_wait(sm.bar(kBarDrain), 0, sm.abort_flag, p.err, false);
}

// Output MMA: O^T block j += V^T_j P~^T, V^T_j = latent unit j of the tile read
// MN-major from its V-ring slot, P~ the weights as two e4m3 terms stacked as
// 2N rows of 128 tokens (K-major), 32 tokens per instruction; the epilogue
// adds the block's two column halves.  Unit by unit: each unit's four
// instructions are issued as soon as it has landed, and its V-ring slot is
// handed back as soon as they complete, so the V producer reloads the next
// tile's units one at a time.  (Waiting for all four and issuing them
// interleaved across the O^T blocks measured 1.4 us slower at 16 columns
// and 3.8 us at 32.)
template <int N, int SQ>
__device__ void output_mma_warp_f8(const DecodeParams &p, const Range &w, const Smem &sm, uint32_t tmem)
{
    using C = Cfg<N, SQ>;
    constexpr uint32_t idO = ptx::idesc_e4m3_f32(128, 2 * N, true, false);  // V^T MN-major, P~^T K-major
    constexpr uint32_t RV = f8_vring<N>();
    const uint32_t vbase = sm.ring + static_cast<uint32_t>(p.ring) * kF8UnitBytes;
    uint32_t it = 0, vc = 0;
    bool ok = true;
    for (int b = w.b0; b <= w.b1 && ok; ++b) {
        const int L = max(0, __ldg(p.seqlens + b));
        const int nt = tiles_of(L);
        const int tb = (b == w.b0) ? w.t0 : 0;
        const int te = min((b == w.b1) ? w.t1 : nt, nt);
        for (int t = tb; t < te && ok; ++t) {
            const uint32_t pb = it & 1, pu = it >> 1;
            if (!(ok = warp_wait(sm.bar(kBarPFull + pb), pu & 1, sm.abort_flag, p.err))) break;
            ptx::tc_fence_after();
            const uint32_t pa = sm.p + pb * 2 * C::QCHUNK;
#pragma unroll 1
            for (int j = 0; j < 4 && ok; ++j) {
                const uint32_t v = vc + j;
                const int slot = static_cast<int>(v % RV);
                if (!(ok = warp_wait(sm.bar(kBarVFull + slot), (v / RV) & 1, sm.abort_flag, p.err))) break;
                ptx::tc_fence_after();
                const uint32_t a0 = vbase + slot * kF8UnitBytes;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    ptx::mma_e4m3_ss_elect(tmem + j * 2 * N, ptx::desc_sw128(a0 + 4096u * kk, 8192, 1024),
                                           ptx::desc_sw128(pa + 32u * kk, 16, 1024), idO, (t != tb) || kk != 0);
                ptx::mma_commit_elect(sm.bar(kBarVEmpty + slot));
            }
            if (!ok) break;
            ptx::mma_commit_elect(sm.bar(kBarPEmpty + pb));
            vc += 4;
            ++it;
        }
    }
    ptx::mma_commit_elect(sm.bar(kBarDrainO));
    warp_wait(sm.bar(kBarDrainO), 0, sm.abort_flag, p.err, false);
}

// FP8 cache: the V producer (the first transposer warp, idle otherwise).
// Walks the same ranges, tiles and page-table windows as the producer and
// loads each tile's four latent units again into the V ring; the producer's
// load of the same bytes has normally just brought them into L2, so the HBM
// traffic stays one read.
template <int N, int SQ>
__device__ void v_producer_warp(const DecodeParams &p, const Range &w, const Smem &sm, const CUtensorMap *kv_map)
{
    constexpr uint32_t RV = f8_vring<N>();
    const int lane = threadIdx.x & 31;
    const uint32_t vbase = sm.ring + static_cast<uint32_t>(p.ring) * kF8UnitBytes;
    uint32_t vc = 0;  // V-ring slot uses so far
    bool ok = true;
    for (int b = w.b0; b <= w.b1 && ok; ++b) {
        const int tb = (b == w.b0) ? w.t0 : 0;
        const int32_t *bt = p.block_table + static_cast<int64_t>(b) * p.max_blocks;
        int win = 2 * tb;
        const int raw_cur = table_entry(bt, win, p, lane);
        const int raw_nxt = table_entry(bt, win + 32, p, lane);
        const int L = max(0, __ldg(p.seqlens + b));
        const int nt = tiles_of(L);
        const int te = min((b == w.b1) ? w.t1 : nt, nt);
        if (tb >= te) continue;
        const int npages = (L + kPage - 1) / kPage;
        int cur = checked_page(raw_cur, win, npages, p, lane);
        int nxt = checked_page(raw_nxt, win + 32, npages, p, lane);
        for (int t = tb; t < te && ok; ++t) {
            if (2 * t >= win + 32) {
                win += 32;
                cur = nxt;
                nxt = load_pages(bt, win + 32, npages, p, lane);
            }
            const int phys0 = __shfl_sync(0xffffffffu, cur, 2 * t - win);
            const int phys1 = __shfl_sync(0xffffffffu, cur, 2 * t + 1 - win);
            const bool live1 = (t * kTile + kPage) < L;
            const uint32_t b8 = live1 ? 2 * kF8Half : kF8Half;
#pragma unroll 1
            for (int j = 0; j < 4; ++j) {
                const uint32_t v = vc + j;
                const int slot = static_cast<int>(v % RV);
                if (!warp_wait(sm.bar(kBarVEmpty + slot), ((v / RV) & 1) ^ 1, sm.abort_flag, p.err)) {
                    ok = false;
                    vc += j;
                    break;
                }
                ptx::mbar_arrive_expect_tx_elect(sm.bar(kBarVFull + slot), b8);
                const uint32_t dst = vbase + slot * kF8UnitBytes;
                ptx::tma_load_3d_elect(dst, kv_map, sm.bar(kBarVFull + slot), 128 * j, 0, phys0);
                if (live1) ptx::tma_load_3d_elect(dst + kF8Half, kv_map, sm.bar(kBarVFull + slot), 128 * j, 0, phys1);
            }
            if (ok) vc += 4;
        }
    }
    if (!ok) {
        // Let every load this warp issued land before the CTA exits.
        const uint32_t first = vc > RV ? vc - RV : 0;
        for (uint32_t v = first; v < vc; ++v)
            warp_wait(sm.bar(kBarVFull + static_cast<int>(v % RV)), (v / RV) & 1, sm.abort_flag, p.err, false);
    }
}

// -- transposer: 4 warps copy V(t) into the TMEM ring as V^T ----------------
// Warp q owns TMEM lanes 32q..32q+31, i.e. latent dims 128j + 32q + (0..31)
// of every 128-dim block j: half of chunk 2j + q/2.  Per 16 dims x 16 tokens
// one ldmatrix.x4.trans feeds one tcgen05.st.16x256b.
template <int N, int SQ, bool F8>
__device__ void transposer_warps(const DecodeParams &p, const Range &w, const Smem &sm, uint32_t tmem)
{
    using C = Cfg<N, SQ>;
    constexpr uint32_t NVT = C::NVT;
    if constexpr (F8) return;  // the FP8 output MMA reads V^T from the ring
    const uint32_t R = static_cast<uint32_t>(p.ring);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = warp & 3;
    uint32_t cc = 0, v = 0;
    bool ok = true;
    // ldmatrix row addresses: lane -> (matrix mi, row rr).  Matrices 0 and 2
    // take tokens {0,1,4,5,8,9,12,13} of a 16-token group, matrices 1 and 3
    // tokens {2,3,6,7,10,11,14,15}: thread t then receives token pairs
    // (4(t%4), 4(t%4)+1) and (4(t%4)+2, 4(t%4)+3), which the 16x256b store puts
    // in TMEM columns 2(t%4) and 2(t%4)+1 -- tokens in natural order.
    const int mi = lane >> 3, rr = lane & 7;
    const int tok_in = 4 * (rr >> 1) + (rr & 1) + 2 * (mi & 1);  // token within a 16-token group
    const int dim_in = 8 * (mi >> 1);                             // dim offset within a 16-dim half
    for (int b = w.b0; b <= w.b1 && ok; ++b) {
        const int L = max(0, __ldg(p.seqlens + b));
        const int nt = tiles_of(L);
        const int tb = (b == w.b0) ? w.t0 : 0;
        const int te = min((b == w.b1) ? w.t1 : nt, nt);
        for (int t = tb; t < te; ++t) {
            const int valid = L - t * kTile;  // tokens of this tile inside the sequence
            // Warp q's share of block j: 16 ldmatrix.x4 = 64 registers.  All
            // 16 loads of a block are in flight together, and the next
            // block's loads are issued before this block is stored, so the
            // shared-memory latency is paid about once per block.
            auto wait_chunk = [&](int j, uint32_t &slot_out) -> bool {
                const int c = 2 * j + (q >> 1);
                const uint32_t u = cc + c / C::CPS;
                slot_out = u % R;
                return warp_wait(sm.bar(kBarFull + static_cast<int>(slot_out)), (u / R) & 1, sm.abort_flag, p.err);
            };
            auto load_chunk = [&](int j, uint32_t slot_id, uint32_t (&r)[64]) {
                const int c = 2 * j + (q >> 1);
                const uint32_t sbase = sm.slot(static_cast<int>(slot_id)) + (c % C::CPS) * kChunkBytes;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int dc = 32 * (q & 1) + 16 * h + dim_in;  // dim within the chunk
#pragma unroll
                    for (int gi = 0; gi < 8; ++gi) {
                        const int tok = 16 * gi + tok_in;
                        const int o = 32 * h + 4 * gi;
                        ptx::ldsm_x4_trans(sbase + tok * 128u + ((((dc >> 3) ^ (tok & 7))) << 4), r[o], r[o + 1],
                                           r[o + 2], r[o + 3]);
                    }
                }
            };
            // The slot is released as soon as this warp's loads of it have
            // returned, so the ring can refill while this warp waits for a
            // free V^T block.  Each lane stores a value computed from every
            // load of the block (so the store cannot complete before the
            // loads do); the arrive, after a proxy fence, orders that store
            // before the producer's next TMA write to the slot.
            auto release = [&](uint32_t slot_id, const uint32_t (&r)[64]) {
                uint32_t x = 0;
#pragma unroll
                for (int i = 0; i < 16; ++i) x |= r[4 * i];
                ptx::st_shared_b32(sm.scratch + 4u * (32u * q + static_cast<uint32_t>(lane)), x);
                __syncwarp();
                if (lane == 0) {
                    ptx::fence_proxy_async_smem();
                    ptx::mbar_arrive(sm.bar(kBarEmpty + static_cast<int>(slot_id)));
                }
            };
            auto store_chunk = [&](uint32_t vb, uint32_t (&r)[64]) {
                if (valid < kTile) {
                    // tokens past the sequence end: their P is zero, make V^T zero too
#pragma unroll
                    for (int h = 0; h < 2; ++h)
#pragma unroll
                        for (int gi = 0; gi < 8; ++gi)
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const int t0 = 16 * gi + 4 * (lane & 3) + 2 * (i & 1);
                                uint32_t &x = r[32 * h + 4 * gi + i];
                                if (t0 >= valid) x = 0;
                                else if (t0 + 1 >= valid) x &= 0xFFFFu;
                            }
                }
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int gg = 0; gg < 2; ++gg) {
                        uint32_t x[16];
#pragma unroll
                        for (int k = 0; k < 16; ++k) x[k] = r[32 * h + 16 * gg + k];
                        ptx::tmem_st_16x256b_x4(
                            tmem + (static_cast<uint32_t>(32 * q + 16 * h) << 16) + C::VT_COL + 64 * vb + 32 * gg, x);
                    }
            };
            uint32_t ra[64], rb[64];
            uint32_t slot_a = 0, slot_b = 0;
            if (!(ok = wait_chunk(0, slot_a))) break;
            load_chunk(0, slot_a, ra);
            release(slot_a, ra);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t(&cur)[64] = (j & 1) ? rb : ra;
                uint32_t(&nxt)[64] = (j & 1) ? ra : rb;
                uint32_t &slot_nxt = (j & 1) ? slot_a : slot_b;
                if (j < 3) {
                    if (!(ok = wait_chunk(j + 1, slot_nxt))) break;
                    load_chunk(j + 1, slot_nxt, nxt);
                    release(slot_nxt, nxt);
                }
                // ring block free: the output MMA that read it last is complete
                const uint32_t vb = v % NVT, vu = v / NVT;
                if (vu >= 1 && !(ok = warp_wait(sm.bar(kBarVtEmpty + vb), (vu & 1) ^ 1, sm.abort_flag, p.err)))
                    break;
                ptx::tc_fence_after();
                store_chunk(vb, cur);
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(sm.bar(kBarVtFull + vb));
                ++v;
            }
            if (!ok) break;
            cc += C::SPT;
        }
    }
}

// -- softmax / epilogue: 4 warps over the 128 token rows of S^T --------------
// S^T is read in the tensor-core fragment layout (tcgen05.ld 16x256b): in
// each 16-row half hf of its warp's 32 rows, thread t holds rows t/4 and
// t/4 + 8 for the two columns 2(t%4), 2(t%4)+1 of every 8-column group, so a
// thread owns N/4 columns and 4 token rows.  P^T goes to shared memory with
// stmatrix.trans straight from that layout (8 tokens x 2 bytes per row).
//
// Scores are kept in the log2 domain relative to a per-column reference max
// mu.  A tile only moves mu -- with an exact column max over the tile, a
// rescale of the running sums and of O^T -- when some score exceeds mu by more
// than 2^kTau (and always on the first tile of a range); otherwise its
// weights 2^(s - mu) are at most 2^kTau and nothing is rescaled.  Every weight
// of a column is taken relative to the same mu as its sum, so the result is
// the same softmax.
template <int N, int SQ, bool F8>
__device__ void softmax_warps(const DecodeParams &p, const Range &w, int g, const Smem &sm, uint32_t tmem)
{
    using C = Cfg<N, SQ>;
    constexpr int HG = C::HG;
    constexpr int NCH = C::NCH;
    constexpr int NG = N / 8;             // 8-column groups
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wq = warp & 3;              // TMEM lane quadrant this warp may access
    const int stid = threadIdx.x - 64;    // 0..127 within the softmax group
    const int c2 = 2 * (lane & 3);        // this thread's first column in each group
    const int r8 = lane >> 2;             // its token row within an 8-row block
    const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
    // stmatrix: lanes 8i..8i+7 address matrix i = (token block i & 1, group offset i >> 1)
    const int st_blk = (lane >> 3) & 1, st_go = lane >> 4, st_row = lane & 7;
    const float NEG_INF = -INFINITY;
    uint32_t it = 0;   // tiles processed
    bool ok = true;

    // FP8 cache: at the start of each range these warps write q as two e4m3
    // terms for the score MMA.  Row n of q (576 bf16 values, 8 significant
    // bits each) is scaled by a power of two 2^a_n that puts its largest
    // magnitude in [128, 256), then hi = e4m3(x) and lo = e4m3(x - hi): x - hi
    // has at most four significant bits, so hi + lo = x exactly unless lo
    // falls below the e4m3 normal range (|x| < 2^-2, i.e. 2^-10 of the row's
    // largest value), where lo keeps its bits down to 2^-9.  The score
    // columns are multiplied back by 2^-a_n (Smem::tscale[n]).  Row n has
    // 128 / N threads (one warp holds whole rows); of each unit's eight
    // 16-column groups a thread takes 8 N / 128 (groups 36-39, past column
    // 575, are the zero fill the rope unit's upper half meets).  The bf16 q
    // lies in the same bytes (nine chunks of 64 columns, N rows x 128 B
    // each); unit u's hi and lo tiles cover chunks 2u and 2u + 1, and row n of
    // them only row n of those chunks, which the row's threads read before
    // any of them writes.
    constexpr int TPR = 128 / N;  // threads per q row
    constexpr int GPU = 8 / TPR;  // 16-column groups per unit and thread
    uint32_t qsplits = 0;
    auto split_q = [&]() -> bool {
        const bool okq = wait_bounded(sm.bar(kBarQFull), qsplits & 1, sm.abort_flag, p.err);
        ++qsplits;
        const int n = stid / TPR, part = stid % TPR;
        const uint32_t qs = sm.q;
        auto load16 = [&](int gq, float (&v)[16]) {
            const int c = gq >> 2, u0 = (gq & 3) * 2;
            const uint32_t rowa = qs + c * C::QCHUNK + n * 128u;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const uint4 x = ptx::ld_shared_v4(rowa + ((static_cast<uint32_t>(u0 + hh) ^ (n & 7)) << 4));
                const uint32_t wv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    v[8 * hh + 2 * e] = __uint_as_float(wv[e] << 16);
                    v[8 * hh + 2 * e + 1] = __uint_as_float(wv[e] & 0xFFFF0000u);
                }
            }
        };
        float mx = 0.f;
#pragma unroll 1
        for (int u = 0; u < kF8Units; ++u)
#pragma unroll
            for (int e = 0; e < GPU; ++e) {
                const int gq = 8 * u + part + TPR * e;
                if (gq >= 36) continue;
                float v[16];
                load16(gq, v);
#pragma unroll
                for (int i = 0; i < 16; ++i) mx = fmaxf(mx, fabsf(v[i]));
            }
#pragma unroll
        for (int o = 1; o < TPR; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        int ex = 0;
        frexpf(mx, &ex);  // mx < 2^ex
        const float up = ldexpf(1.f, 8 - ex);
#pragma unroll 1
        for (int u = 0; u < kF8Units; ++u) {
            float v[GPU][16];
#pragma unroll
            for (int e = 0; e < GPU; ++e) {
                const int gq = 8 * u + part + TPR * e;
                if (gq < 36) {
                    load16(gq, v[e]);
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[e][i] = 0.f;
                }
            }
            __syncwarp();  // the row's bf16 values of unit u are in registers
#pragma unroll
            for (int e = 0; e < GPU; ++e) {
                const int gq = 8 * u + part + TPR * e;
                uint32_t hw[4], lw[4];
#pragma unroll
                for (int e4 = 0; e4 < 4; ++e4) {
                    uint32_t hb[2], lb[2];
#pragma unroll
                    for (int e2 = 0; e2 < 2; ++e2) {
                        const float x0 = v[e][4 * e4 + 2 * e2] * up, x1 = v[e][4 * e4 + 2 * e2 + 1] * up;
                        hb[e2] = ptx::f32x2_to_e4m3x2(x0, x1);
                        float h0, h1;
                        ptx::e4m3x2_to_f32x2(hb[e2], h0, h1);
                        lb[e2] = ptx::f32x2_to_e4m3x2(x0 - h0, x1 - h1);
                    }
                    hw[e4] = hb[0] | (hb[1] << 16);
                    lw[e4] = lb[0] | (lb[1] << 16);
                }
                const uint32_t at = qs + u * C::QS8_UNIT + n * 128u +
                                    ((static_cast<uint32_t>(gq & 7) ^ static_cast<uint32_t>(n & 7)) << 4);
                ptx::st_shared_v4(at, hw[0], hw[1], hw[2], hw[3]);
                ptx::st_shared_v4(at + N * 128u, lw[0], lw[1], lw[2], lw[3]);
            }
        }
        if (part == 0) sm.tscale[n] = ldexpf(1.f, ex - 8);
        ptx::fence_proxy_async_smem();
        ptx::named_bar_sync(1, 128);
        if (lane == 0) ptx::mbar_arrive(sm.bar(kBarQsFull));
        return okq;
    };

    for (int b = w.b0; b <= w.b1 && ok; ++b) {
        const int L = max(0, __ldg(p.seqlens + b));
        const int nt = tiles_of(L);
        const int tb = (b == w.b0) ? w.t0 : 0;
        const int te = min((b == w.b1) ? w.t1 : nt, nt);
        if (tb >= te) continue;
        const int split = (b == w.b0) ? w.split0 : 0;
        const int nvis0 = L - SQ + 1;  // query position i sees tokens < nvis0 + i (none when that is <= 0)
        float l[NG][2], mu[NG][2];             // this thread's columns: running sums, reference max
#pragma unroll
        for (int gi = 0; gi < NG; ++gi) l[gi][0] = l[gi][1] = mu[gi][0] = mu[gi][1] = 0.f;
        bool wait_ok = true;  // a failed wait is carried to the next agreement point
        float qsc[NG][2];     // FP8: 2^-a of this thread's columns
        if constexpr (F8) {
            wait_ok = split_q() && wait_ok;
#pragma unroll
            for (int gi = 0; gi < NG; ++gi) {
                qsc[gi][0] = sm.tscale[8 * gi + c2];
                qsc[gi][1] = sm.tscale[8 * gi + c2 + 1];
            }
        }

        for (int t = tb; t < te; ++t) {
            const uint32_t sb = it % C::NS, su = it / C::NS;
            wait_ok = wait_bounded(sm.bar(kBarSFull + sb), su & 1, sm.abort_flag, p.err) && wait_ok;
            ptx::tc_fence_after();
            uint32_t raw[2][4 * NG];
            if constexpr (F8) {  // the hi and lo halves of S^T
                uint32_t lo[2][4 * NG];
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const uint32_t ta = tmem + (static_cast<uint32_t>(32 * wq + 16 * hf) << 16) + C::S_COL8 + sb * 2 * N;
                    ptx::tmem_ld_16x256b(ta, raw[hf]);
                    ptx::tmem_ld_16x256b(ta + N, lo[hf]);
                }
                ptx::tmem_wait_ld();
#pragma unroll
                for (int hf = 0; hf < 2; ++hf)
#pragma unroll
                    for (int i = 0; i < 4 * NG; ++i)
                        raw[hf][i] = __float_as_uint(__uint_as_float(raw[hf][i]) + __uint_as_float(lo[hf][i]));
            } else {
#pragma unroll
                for (int hf = 0; hf < 2; ++hf)
                    ptx::tmem_ld_16x256b(tmem + (static_cast<uint32_t>(32 * wq + 16 * hf) << 16) + C::S_COL + sb * N,
                                         raw[hf]);
                ptx::tmem_wait_ld();
            }
            // S^T(it) is in registers: its TMEM buffer may be overwritten
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(sm.bar(kBarSEmpty + sb));

            // pass 1: masked log2-domain scores relative to mu
            const bool first = (t == tb);
            const int tok0 = t * kTile + 32 * wq + r8;
            // FP8 cache: the scales of this thread's four token rows (0 for rows
            // past the sequence's end), from the buffer that landed with the
            // tile's first unit (which the score MMA waited for).  A token's
            // weight in O is 2^(x - mu) tsc with x its log2-domain score;
            // the reference max mu follows x + log2|tsc|, so that weight is
            // at most 2^kTau8 in magnitude.  lgt = log2|tsc| (0 where tsc is 0)
            // and sgt = the sign of tsc (0 where tsc is 0).
            float tsc[2][2] = {{1.f, 1.f}, {1.f, 1.f}}, lgt[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
            float sgt[2][2] = {{1.f, 1.f}, {1.f, 1.f}};
            if constexpr (F8) {
                const uint32_t sbuf = sm.f8 + (it % kRawScBufs) * 512u;
#pragma unroll
                for (int hf = 0; hf < 2; ++hf)
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj) {
                        const int row = 32 * wq + r8 + 16 * hf + 8 * jj;
                        const float x = (tok0 + 16 * hf + 8 * jj < L) ? ptx::ld_shared_f32(sbuf + 4u * row) : 0.f;
                        tsc[hf][jj] = x;
                        lgt[hf][jj] = x != 0.f ? __log2f(fabsf(x)) : 0.f;
                        sgt[hf][jj] = x > 0.f ? 1.f : (x < 0.f ? -1.f : 0.f);
                    }
            }
            float d[2][NG][4];
            bool flag = first || !wait_ok;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf)
#pragma unroll
                for (int gi = 0; gi < NG; ++gi)
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int tok = tok0 + 16 * hf + 8 * (j >> 1);
                        // column n = 8 gi + c2 + (j & 1) belongs to query position
                        // (8 gi) / HG (HG is a multiple of 8), which sees the first
                        // L - SQ + 1 + i tokens
                        const int qi = (8 * gi) / HG;
                        const bool vis = tok < nvis0 + qi;
                        float s = __uint_as_float(raw[hf][4 * gi + j]);
                        if constexpr (F8) {
                            s *= tsc[hf][j >> 1] * qsc[gi][j & 1];
                            d[hf][gi][j] = vis ? fmaf(s, p.scale_log2, lgt[hf][j >> 1] - mu[gi][j & 1]) : NEG_INF;
                            flag = flag || (d[hf][gi][j] > kTau8);
                        } else {
                            d[hf][gi][j] = vis ? fmaf(s, p.scale_log2, -mu[gi][j & 1]) : NEG_INF;
                            flag = flag || (d[hf][gi][j] > kTau);
                        }
                    }
            __syncwarp();
            if (ptx::named_bar_or(1, 128, flag)) {
                if (!(ok = ptx::named_bar_and(1, 128, wait_ok))) break;
                // exact column max of this tile (relative to mu): over the
                // thread's 4 rows, the 8 lanes sharing its columns, the 4 warps
                float cm[NG][2];
#pragma unroll
                for (int gi = 0; gi < NG; ++gi)
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj) {
                        float m = fmaxf(fmaxf(d[0][gi][jj], d[0][gi][jj + 2]), fmaxf(d[1][gi][jj], d[1][gi][jj + 2]));
                        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
                        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
                        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
                        cm[gi][jj] = m;
                    }
                if (r8 == 0) {
#pragma unroll
                    for (int gi = 0; gi < NG; ++gi)
                        *reinterpret_cast<float2 *>(sm.red + wq * N + 8 * gi + c2) = make_float2(cm[gi][0], cm[gi][1]);
                }
                __syncwarp();
                ptx::named_bar_sync(1, 128);
                // shift of column n: on the first tile the exact max (none if
                // the column saw no token), afterwards only upwards
                if (stid < N) {
                    const int n = stid;
                    const float x = fmaxf(fmaxf(sm.red[n], sm.red[N + n]), fmaxf(sm.red[2 * N + n], sm.red[3 * N + n]));
                    float sh;
                    if constexpr (F8)  // FP8: the tile's largest weight becomes 2^kLift8 (see kLift8)
                        sh = first ? (x == NEG_INF ? 0.f : x - kLift8) : fmaxf(x - kLift8, 0.f);
                    else
                        sh = first ? (x == NEG_INF ? 0.f : x) : fmaxf(x, 0.f);
                    sm.shift[n] = sh;
                    sm.mu[n] = (first ? 0.f : sm.mu[n]) + sh;
                }
                __syncwarp();
                ptx::named_bar_sync(1, 128);
#pragma unroll
                for (int gi = 0; gi < NG; ++gi) {
                    const float2 s2 = *reinterpret_cast<const float2 *>(sm.shift + 8 * gi + c2);
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj) {
                        const float sh = jj ? s2.y : s2.x;
                        mu[gi][jj] += sh;
                        if (!first) l[gi][jj] *= ptx::ex2_approx(-sh);
#pragma unroll
                        for (int hf = 0; hf < 2; ++hf) {
                            d[hf][gi][jj] -= sh;
                            d[hf][gi][jj + 2] -= sh;
                        }
                    }
                }
                if (!first) {
                    // O^T is rescaled once the previous tile's output MMA is complete
                    const uint32_t pp = it - 1;
                    wait_ok = wait_bounded(sm.bar(kBarPEmpty + (pp & 1)), (pp >> 1) & 1, sm.abort_flag, p.err) &&
                              wait_ok;
                    ptx::tc_fence_after();
#pragma unroll 1
                    for (int ch = 0; ch < NCH; ++ch) {
                        float a[16];
                        const float4 *s4 = reinterpret_cast<const float4 *>(sm.shift + 16 * ch);
#pragma unroll
                        for (int e4 = 0; e4 < 4; ++e4) {
                            const float4 v4 = s4[e4];
                            a[4 * e4 + 0] = ptx::ex2_approx(-v4.x);
                            a[4 * e4 + 1] = ptx::ex2_approx(-v4.y);
                            a[4 * e4 + 2] = ptx::ex2_approx(-v4.z);
                            a[4 * e4 + 3] = ptx::ex2_approx(-v4.w);
                        }
#pragma unroll 1
                        for (int j = 0; j < (F8 ? 8 : 4); ++j) {  // FP8: both halves of the 4 blocks
                            float x[16];
                            const uint32_t ta = tmem + lane_base + j * N + ch * 16;
                            ptx::tmem_ld16(ta, x);
                            ptx::tmem_wait_ld();
#pragma unroll
                            for (int e = 0; e < 16; ++e) x[e] *= a[e];
                            ptx::tmem_st16(ta, x);
                        }
                    }
                    ptx::tmem_wait_st();
                }
            }

            // pass 2: weights -> P^T and the running sums, into P buffer it & 1
            // once the output MMA of tile it - 2 is done
            if (it >= 2)
                wait_ok = wait_bounded(sm.bar(kBarPEmpty + (it & 1)), ((it >> 1) & 1) ^ 1, sm.abort_flag, p.err) &&
                          wait_ok;
            const uint32_t pbuf = sm.p + (it & 1) * 2 * C::QCHUNK;
            if constexpr (F8) {
                // FP8: l takes 2^(x - mu); O takes w = 2^(x - mu) tsc as two
                // e4m3 terms, hi = e4m3(w) and lo = e4m3(w - hi) (8 significant
                // bits together, like bf16), written as P~^T (row n, token k at
                // n * 128 + ((k / 16) ^ (n % 8)) * 16 + k % 16; hi rows n, lo rows
                // N + n)
#pragma unroll
                for (int hf = 0; hf < 2; ++hf)
#pragma unroll
                    for (int gi = 0; gi < NG; ++gi)
#pragma unroll
                        for (int jh = 0; jh < 2; ++jh) {  // token row r8 + 16 hf + 8 jh, columns n, n + 1
                            const float dl = d[hf][gi][2 * jh], dr = d[hf][gi][2 * jh + 1];
                            l[gi][0] += ptx::ex2_approx(dl - lgt[hf][jh]);
                            l[gi][1] += ptx::ex2_approx(dr - lgt[hf][jh]);
                            const float w0 = ptx::ex2_approx(dl) * sgt[hf][jh];
                            const float w1 = ptx::ex2_approx(dr) * sgt[hf][jh];
                            const uint32_t hb = ptx::f32x2_to_e4m3x2(w0, w1);
                            float h0, h1;
                            ptx::e4m3x2_to_f32x2(hb, h0, h1);
                            const uint32_t lb = ptx::f32x2_to_e4m3x2(w0 - h0, w1 - h1);
                            const int k = 32 * wq + r8 + 16 * hf + 8 * jh;
                            const int n = 8 * gi + c2;
                            const uint32_t a0 = pbuf + n * 128u +
                                                ((static_cast<uint32_t>(k >> 4) ^ static_cast<uint32_t>(n & 7)) << 4) +
                                                static_cast<uint32_t>(k & 15);
                            const uint32_t a1 = pbuf + (n + 1) * 128u +
                                                ((static_cast<uint32_t>(k >> 4) ^ static_cast<uint32_t>((n + 1) & 7)) << 4) +
                                                static_cast<uint32_t>(k & 15);
                            ptx::st_shared_u8(a0, hb & 0xFFu);
                            ptx::st_shared_u8(a1, hb >> 8);
                            ptx::st_shared_u8(a0 + N * 128u, lb & 0xFFu);
                            ptx::st_shared_u8(a1 + N * 128u, lb >> 8);
                        }
                // Rows past the sequence's end in its last tile hold whatever the
                // cache (or an earlier unit) left there, NaN codes included; their
                // weights are zero, and the V^T the output MMA reads must be finite
                // too: once the tile's four V-ring units have landed, this thread
                // zeroes its row of them.
                const int valid = L - t * kTile;  // the same in every thread
                if (valid < kTile) {
                    constexpr uint32_t RV = f8_vring<N>();
                    const uint32_t vbase = sm.ring + static_cast<uint32_t>(p.ring) * kF8UnitBytes;
                    const int r = 32 * wq + lane;
#pragma unroll 1
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t v = 4 * it + j;
                        const int slot = static_cast<int>(v % RV);
                        wait_ok = warp_wait(sm.bar(kBarVFull + slot), (v / RV) & 1, sm.abort_flag, p.err) && wait_ok;
                        if (r >= valid) {
                            const uint32_t ra = vbase + slot * kF8UnitBytes + r * 128u;
#pragma unroll
                            for (int c = 0; c < 8; ++c) ptx::st_shared_v4(ra + 16u * c, 0u, 0u, 0u, 0u);
                        }
                    }
                }
            } else {
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    uint32_t pk[NG][2];
#pragma unroll
                    for (int gi = 0; gi < NG; ++gi) {
                        const float p0 = ptx::ex2_approx(d[hf][gi][0]);  // masked entries: 2^-inf = 0
                        const float p1 = ptx::ex2_approx(d[hf][gi][1]);
                        const float p2 = ptx::ex2_approx(d[hf][gi][2]);
                        const float p3 = ptx::ex2_approx(d[hf][gi][3]);
                        l[gi][0] += p0 + p2;
                        l[gi][1] += p1 + p3;
                        pk[gi][0] = ptx::pack_bf16x2(p0, p1);  // token row r8
                        pk[gi][1] = ptx::pack_bf16x2(p2, p3);  // token row r8 + 8
                    }
                    // P^T rows n, K positions = tokens of the tile (natural order)
                    const int kb = 32 * wq + 16 * hf + 8 * st_blk;  // first token of this lane's matrix
                    const uint32_t kbase = pbuf + (kb >> 6) * C::QCHUNK;
                    const uint32_t kchunk = static_cast<uint32_t>((kb & 63) >> 3);
#pragma unroll
                    for (int gp = 0; gp < NG / 2; ++gp) {
                        const int n = 8 * (2 * gp + st_go) + st_row;
                        const uint32_t addr = kbase + n * 128u + ((kchunk ^ static_cast<uint32_t>(n & 7)) << 4);
                        ptx::stsm_x4_trans(addr, pk[2 * gp][0], pk[2 * gp][1], pk[2 * gp + 1][0], pk[2 * gp + 1][1]);
                    }
                }
            }
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            ptx::mbar_arrive(sm.bar(kBarPFull + (it & 1)));
            ++it;
        }
        if (!ok) break;
        // ---- epilogue of this range: its last output MMA must be complete
        const uint32_t pp = it - 1;
        wait_ok = wait_bounded(sm.bar(kBarPEmpty + (pp & 1)), (pp >> 1) & 1, sm.abort_flag, p.err) && wait_ok;
        __syncwarp();
        if (!(ok = ptx::named_bar_and(1, 128, wait_ok))) break;
        ptx::tc_fence_after();
        range_epilogue<N, SQ, F8>(p, sm, tmem, b, split, g, l);
    }
}

// ============================================================== kernel
// Prologue: shared-memory carve-up, barrier initialisation and TMEM
// allocation (none of which reads an input), then -- once the previous grid
// of the stream has completed, when launched as its programmatic dependent --
// the schedule check.  Returns false (uniformly) when this CTA has no work;
// TMEM is allocated either way and released by decode_teardown.
template <int N, int SQ, bool F8>
__device__ __forceinline__ bool decode_setup(const DecodeParams &p, const CUtensorMap *kv_map,
                                             const CUtensorMap *q_map, const CUtensorMap *sc_map, uint8_t *smem_raw,
                                             Smem &sm, Range &w, uint32_t &tmem)
{
    using C = Cfg<N, SQ>;
    const uint32_t raw = ptx::smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - raw);
    sm.ring = base;
    sm.slot_bytes = F8 ? kF8UnitBytes : C::SLOT_BYTES;
    uint32_t off = p.ring * (F8 ? kF8UnitBytes : C::SLOT_BYTES);
    if constexpr (F8) off += f8_vring<N>() * kF8UnitBytes;
    sm.f8 = base + off;  // FP8: the unit ring, the V ring, the token scales, then q (split in place) and P~^T
    if constexpr (F8) off += kRawScBytes;
    sm.q = base + off;
    constexpr uint32_t qreg = F8 ? C::QS8 : C::QBYTES;
    sm.p = sm.q + qreg;
    uint8_t *misc = gbase + off + qreg + C::PBYTES;
    sm.bars = ptx::smem_addr(misc);
    sm.red = reinterpret_cast<float *>(misc + kMiscRedOffset);
    sm.lred = sm.red + 4 * N;
    sm.mu = sm.lred + 4 * N;
    sm.shift = sm.mu + N;
    sm.tmem_holder = reinterpret_cast<uint32_t *>(sm.shift + N);
    sm.abort_flag = reinterpret_cast<volatile int *>(sm.tmem_holder + 1);
    sm.scratch = ptx::smem_addr(sm.tmem_holder + 4);
    sm.tscale = reinterpret_cast<float *>(misc + misc_bytes<N>());  // FP8 only: q scales, past the misc region

    const int warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) {
        for (int s = 0; s < p.ring; ++s) {
            ptx::mbar_init(sm.bar(kBarFull + s), 1);
            // FP8: a unit's slot is free after the score MMA
            ptx::mbar_init(sm.bar(kBarEmpty + s), F8 ? 1 : C::EMPTY_ARRIVALS);
        }
        if constexpr (F8) {
            ptx::mbar_init(sm.bar(kBarQsFull), 4);  // one arrival per softmax warp
            for (int i = 0; i < f8_vring<N>(); ++i) {
                ptx::mbar_init(sm.bar(kBarVFull + i), 1);
                ptx::mbar_init(sm.bar(kBarVEmpty + i), 1);
            }
        } else {
            // (unused by the bf16 instances; kept so their set-up is unchanged)
            for (int i = 0; i < 4; ++i) {
                ptx::mbar_init(sm.bar(kBarF8Full + i), 1);
                ptx::mbar_init(sm.bar(kBarF8Full + 4 + i), 4);
            }
            for (int i = 0; i < kScBufs; ++i) {
                ptx::mbar_init(sm.bar(kBarF8Full + 8 + i), 4);
                ptx::mbar_init(sm.bar(kBarF8Full + 8 + kScBufs + i), 4);
            }
        }
        ptx::mbar_init(sm.bar(kBarQFull), 1);
        ptx::mbar_init(sm.bar(kBarQEmpty), 1);
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(sm.bar(kBarSFull + i), 1);
            ptx::mbar_init(sm.bar(kBarSEmpty + i), 4);
            ptx::mbar_init(sm.bar(kBarPFull + i), 128);
            ptx::mbar_init(sm.bar(kBarPEmpty + i), 1);
        }
        for (int i = 0; i < kMaxVt; ++i) {
            ptx::mbar_init(sm.bar(kBarVtFull + i), 4);
            ptx::mbar_init(sm.bar(kBarVtEmpty + i), 1);
        }
        ptx::mbar_init(sm.bar(kBarDrain), 1);
        ptx::mbar_init(sm.bar(kBarDrainO), 1);
        *sm.abort_flag = 0;
        ptx::fence_mbar_init();
        ptx::tma_prefetch_map(kv_map);
        ptx::tma_prefetch_map(q_map);
        if (F8) ptx::tma_prefetch_map(sc_map);
    }
    if (warp == 1) {
        ptx::tmem_alloc(ptx::smem_addr(sm.tmem_holder), C::TMEM_COLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    tmem = *sm.tmem_holder;

    // Everything below reads inputs that earlier kernels of the stream write.
    ptx::griddep_wait();
    const int tuple = blockIdx.x / p.G;
    const int32_t *hdr = p.sched;
    if (hdr[1] != kSchedMagic || hdr[2] != p.B || hdr[3] != p.s_q || hdr[4] != p.H ||
        hdr[5] != p.num_sms || hdr[6] != p.num_tuples || hdr[7] != p.G) {
        if (threadIdx.x == 0) atomicOr(p.err, MLA_DEVERR_SCHEDULE);
        return false;
    }
    const int32_t *e = p.sched + kSchedHeader + tuple * kSchedEntry;
    w = Range{e[0], e[1], e[2], e[3], e[4]};
    if (w.b0 < 0) return false;  // no work for this group
    if (w.b0 >= p.B || w.b1 < w.b0 || w.b1 >= p.B || w.t0 < 0 || w.t1 < 0) {
        if (threadIdx.x == 0) atomicOr(p.err, MLA_DEVERR_SCHEDULE);
        return false;
    }
    return true;
}

template <int N, int SQ>
__device__ __forceinline__ void decode_teardown(uint32_t tmem)
{
    using C = Cfg<N, SQ>;
    ptx::tc_fence_before();
    __syncthreads();
    if ((threadIdx.x >> 5) == 1) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// Warps: 0 producer, 1 score MMA (and TMEM owner), 2-5 softmax + epilogue,
// 6-9 transposer (FP8: 6 the V producer, 7-9 idle), 10 output MMA.
template <int N, int SQ, bool F8>
__global__ void __launch_bounds__(kThreads, 1)
mla_decode_kernel(const __grid_constant__ CUtensorMap kv_map, const __grid_constant__ CUtensorMap q_map,
                  const __grid_constant__ CUtensorMap sc_map, const DecodeParams p)
{
    extern __shared__ uint8_t smem_raw[];
    Smem sm;
    Range w;
    uint32_t tmem;
    ptx::griddep_launch_dependents();
    if (decode_setup<N, SQ, F8>(p, &kv_map, &q_map, &sc_map, smem_raw, sm, w, tmem)) {
        const int warp = threadIdx.x >> 5;
        const int g = blockIdx.x % p.G;
        if (warp == 0) {
            producer_warp<N, SQ, F8>(p, w, g, sm, &kv_map, &q_map, &sc_map);
        } else if (warp == 1) {
            if constexpr (F8) score_mma_warp_f8<N, SQ>(p, w, sm, tmem);
            else score_mma_warp<N, SQ>(p, w, sm, tmem);
        } else if (warp < 6) {
            softmax_warps<N, SQ, F8>(p, w, g, sm, tmem);
        } else if (warp < 10) {
            if constexpr (F8) {
                if (warp == 6) v_producer_warp<N, SQ>(p, w, sm, &kv_map);
            } else {
                transposer_warps<N, SQ, F8>(p, w, sm, tmem);
            }
        } else {
            if constexpr (F8) output_mma_warp_f8<N, SQ>(p, w, sm, tmem);
            else output_mma_warp<N, SQ>(p, w, sm, tmem);
        }
    }
    decode_teardown<N, SQ>(tmem);
}

// =============================================================== combine
// One 128-thread block per output row (b, i, h) of a sequence cut into pieces.
// Each thread owns four latent dims and issues the loads of a batch of
// pieces together.  Two instances: 20 pieces per batch (128 registers, four
// blocks per SM) when the rows fit in one wave -- the ~19 pieces of a
// 64K-context sequence split over 148 SMs in one memory round trip -- and 8
// pieces (64 registers, eight blocks per SM) for many rows of few pieces
// (8192 rows at 128 heads), where resident blocks matter more.  Launched as a
// programmatic dependent of the attention kernel: it may become resident
// early and waits in hardware for that grid to finish.
constexpr int kCombineThreads = 128;

template <int kBatch>
__global__ void __launch_bounds__(kCombineThreads, kBatch > 8 ? 4 : 8)
mla_combine_kernel(const int32_t *__restrict__ split_base, const float *__restrict__ ws_o,
                   const float *__restrict__ ws_lse, int B, int s_q, int H, int HG, int G, int max_pieces,
                   uint16_t *__restrict__ out, float *__restrict__ lse, int32_t *__restrict__ err)
{
    ptx::griddep_wait();       // the attention grid (and its memory) is complete
    const int tid = threadIdx.x;
    const int64_t r = blockIdx.x;
    const int h = static_cast<int>(r % H);
    const int i = static_cast<int>((r / H) % s_q);
    const int b = static_cast<int>(r / (static_cast<int64_t>(H) * s_q));
    const int first = split_base[b];
    const int n = split_base[b + 1] - first;
    if (n == 1) return;  // written directly by the attention kernel
    uint2 *o = reinterpret_cast<uint2 *>(out + r * kDV) + tid;  // four bf16 per thread
    if (n <= 0) {
        *o = make_uint2(0, 0);
        if (tid == 0) lse[r] = -INFINITY;
        return;
    }
    if (first < 0 || (static_cast<int64_t>(first) + n) * G > max_pieces || n > kMaxSms) {
        if (tid == 0) atomicOr(err, MLA_DEVERR_SCHEDULE);
        return;
    }
    const int g = h / HG, hl = h % HG;
    const int64_t row0 = (static_cast<int64_t>(first) * G + g) * s_q * HG + static_cast<int64_t>(i) * HG + hl;
    const int64_t pstride = static_cast<int64_t>(G) * s_q * HG;  // rows between consecutive pieces
    const int64_t step = pstride * kDV / 4;                      // float4s between consecutive pieces
    const float *lp = ws_lse + row0;
    const float4 *sp = reinterpret_cast<const float4 *>(ws_o + row0 * kDV) + tid;
    // Every thread reads the pieces' lse values itself (broadcast loads) with
    // its own partials, a batch at a time, and keeps a running max, so a row
    // of up to kBatch pieces costs one round trip.
    float M = -INFINITY, ssum = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int k0 = 0; k0 < n; k0 += kBatch) {
        float4 x[kBatch];
        float lk[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            lk[u] = -INFINITY;
            if (k0 + u < n) {
                x[u] = *sp;
                lk[u] = *lp;
            }
            sp += step;
            lp += pstride;
        }
        float bm = lk[0];
#pragma unroll
        for (int u = 1; u < kBatch; ++u) bm = fmaxf(bm, lk[u]);
        if (bm > M) {  // new running max: rescale what was summed so far
            const float a = (M == -INFINITY) ? 0.f : expf(M - bm);
            acc.x *= a; acc.y *= a; acc.z *= a; acc.w *= a;
            ssum *= a;
            M = bm;
        }
        if (M == -INFINITY) continue;  // no piece so far saw a token
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            if (k0 + u < n) {
                const float wk = expf(lk[u] - M);  // pieces without tokens: lse = -inf, weight 0
                ssum += wk;
                acc.x += wk * x[u].x;
                acc.y += wk * x[u].y;
                acc.z += wk * x[u].z;
                acc.w += wk * x[u].w;
            }
        }
    }
    if (M == -INFINITY) {  // every piece saw no token
        *o = make_uint2(0, 0);
        if (tid == 0) lse[r] = -INFINITY;
        return;
    }
    const float inv = 1.f / ssum;
    __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
    __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
    uint2 packed;
    packed.x = *reinterpret_cast<uint32_t *>(&lo);
    packed.y = *reinterpret_cast<uint32_t *>(&hi);
    *o = packed;
    if (tid == 0) lse[r] = M + logf(ssum);
}

// ================================================================== host
namespace host {

struct Shape {
    int N, SQ, HG, G;
};

// Query columns per CTA: N = s_q H when that is at most 64, else 64 in
// G = s_q H / 64 head groups of 64 / s_q heads.
bool resolve(int s_q, int H, Shape *s)
{
    if (s_q != 1 && s_q != 2 && s_q != 4 && s_q != 8) return false;
    if (H != 16 && H != 32 && H != 64 && H != 128) return false;
    const int tot = s_q * H;
    s->SQ = s_q;
    if (tot <= 64) {
        s->N = tot;
        s->G = 1;
    } else {
        s->N = 64;
        s->G = tot / 64;
    }
    s->HG = s->N / s_q;
    return true;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct WorkspaceLayout {
    int pieces;
    size_t o_bytes, lse_off, total;
};

WorkspaceLayout layout(int B, int s_q, const Shape &sh, int num_sms)
{
    const int tuples = num_sms / sh.G;
    const size_t pieces = static_cast<size_t>(B + tuples) * sh.G;
    WorkspaceLayout w;
    w.pieces = static_cast<int>(pieces);
    w.o_bytes = align256(pieces * s_q * sh.HG * kDV * sizeof(float));
    w.lse_off = w.o_bytes;
    w.total = w.o_bytes + align256(pieces * s_q * sh.HG * sizeof(float));
    return w;
}

thread_local char g_last_error[256] = "";

mla_status_t cuda_fail(cudaError_t e, const char *what)
{
    snprintf(g_last_error, sizeof g_last_error, "%s: %s", what, cudaGetErrorString(e));
    return MLA_ERR_CUDA;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// Encoded tensor maps, cached by everything that goes into the encoding (the
// tensor's address, shape, strides, box and layout options): a repeated call
// on the same buffers reuses the map instead of encoding it again.  A map
// holds only an address and a shape, so a cached one stays valid for any
// buffer that is later placed at the same address with the same shape.
struct MapKey {
    int dtype, rank, swizzle, promo;
    const void *ptr;
    cuuint64_t dims[3], strides[2];
    cuuint32_t box[3];
};

struct MapEntry {
    bool used;
    MapKey key;
    CUtensorMap map;
};

constexpr int kMapCache = 32;
std::mutex g_map_mutex;
MapEntry g_maps[kMapCache];
int g_map_next = 0;

bool same_key(const MapKey &a, const MapKey &b)
{
    if (a.dtype != b.dtype || a.rank != b.rank || a.swizzle != b.swizzle || a.promo != b.promo || a.ptr != b.ptr)
        return false;
    for (int i = 0; i < a.rank; ++i)
        if (a.dims[i] != b.dims[i] || a.box[i] != b.box[i]) return false;
    for (int i = 0; i + 1 < a.rank; ++i)
        if (a.strides[i] != b.strides[i]) return false;
    return true;
}

// Tiled tensor map of `rank` <= 3 dimensions (element strides 1, no
// interleave, zero fill); returns false with the message set on failure.
bool tensor_map(CUtensorMap *out, const char *what, CUtensorMapDataType dtype, int rank, const void *ptr,
                const cuuint64_t *dims, const cuuint64_t *strides, const cuuint32_t *box, CUtensorMapSwizzle swizzle,
                CUtensorMapL2promotion promo)
{
    MapKey key;
    memset(&key, 0, sizeof key);
    key.dtype = static_cast<int>(dtype);
    key.rank = rank;
    key.swizzle = static_cast<int>(swizzle);
    key.promo = static_cast<int>(promo);
    key.ptr = ptr;
    for (int i = 0; i < rank; ++i) {
        key.dims[i] = dims[i];
        key.box[i] = box[i];
    }
    for (int i = 0; i + 1 < rank; ++i) key.strides[i] = strides[i];
    {
        std::lock_guard<std::mutex> lock(g_map_mutex);
        for (int i = 0; i < kMapCache; ++i)
            if (g_maps[i].used && same_key(g_maps[i].key, key)) {
                *out = g_maps[i].map;
                return true;
            }
    }
    EncodeTiledFn encode = encode_fn();
    if (!encode) {
        snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled unavailable");
        return false;
    }
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = encode(out, dtype, static_cast<cuuint32_t>(rank), const_cast<void *>(ptr), dims, strides, box,
                              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, promo, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled(%s) failed: %d", what, static_cast<int>(r));
        return false;
    }
    std::lock_guard<std::mutex> lock(g_map_mutex);
    MapEntry &e = g_maps[g_map_next];
    g_map_next = (g_map_next + 1) % kMapCache;
    e.used = true;
    e.key = key;
    e.map = *out;
    return true;
}

struct DeviceInfo {
    int smem_optin = 0;
    int major = 0;
    bool attr_set[10] = {};
};

std::mutex g_dev_mutex;
DeviceInfo g_dev[64];

template <int N, int SQ, bool F8>
int kernel_index()
{
    if (F8) return N == 16 ? 7 : (SQ == 1 ? 8 : 9);
    if (N == 16 && SQ == 1) return 0;
    if (N == 32 && SQ == 1) return 1;
    if (N == 32 && SQ == 2) return 2;
    if (N == 64 && SQ == 1) return 3;
    if (N == 64 && SQ == 2) return 4;
    if (N == 64 && SQ == 4) return 5;
    return 6;
}

template <int N, int SQ, bool F8>
int ring_for(int smem_optin, size_t *smem_bytes)
{
    using C = Cfg<N, SQ>;
    const int fixed = static_cast<int>((F8 ? C::QS8 : C::QBYTES) + C::PBYTES + misc_bytes<N>() + 1024 +
                                       (F8 ? kRawScBytes + kQScaleBytes + f8_vring<N>() * kF8UnitBytes : 0));
    const uint32_t slot = F8 ? kF8UnitBytes : C::SLOT_BYTES;
    int R = (smem_optin - fixed) / static_cast<int>(slot);
    if (R > kMaxRing) R = kMaxRing;
    *smem_bytes = static_cast<size_t>(fixed) + static_cast<size_t>(R) * slot;
    return R;
}

template <int N, int SQ, bool F8>
mla_status_t launch_decode(const CUtensorMap &kv_map, const CUtensorMap &q_map, const CUtensorMap &sc_map,
                           DecodeParams prm, int grid, cudaStream_t stream)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= 64) return cuda_fail(cudaErrorInvalidDevice, "device index");
    DeviceInfo info;
    {
        std::lock_guard<std::mutex> lock(g_dev_mutex);
        DeviceInfo &d = g_dev[dev];
        if (d.smem_optin == 0) {
            e = cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
            if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute(smem)");
            e = cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev);
            if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute(cc)");
        }
        info = d;
    }
    if (info.major != 10) {
        snprintf(g_last_error, sizeof g_last_error, "device %d is not sm_100 (compute capability %d.x)", dev,
                 info.major);
        return MLA_ERR_CUDA;
    }
    size_t smem = 0;
    const int R = ring_for<N, SQ, F8>(info.smem_optin, &smem);
    if (R * Cfg<N, SQ>::CPS < kMinRingChunks || (F8 && R < kF8Units)) {
        snprintf(g_last_error, sizeof g_last_error, "not enough shared memory for a %d-chunk ring", kMinRingChunks);
        return MLA_ERR_CUDA;
    }
    const int ki = kernel_index<N, SQ, F8>();
    void (*kernel)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const DecodeParams) =
        mla_decode_kernel<N, SQ, F8>;
    if (!info.attr_set[ki]) {
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
        std::lock_guard<std::mutex> lock(g_dev_mutex);
        g_dev[dev].attr_set[ki] = true;
    }
    prm.ring = R;
    // Programmatic dependent launch: the CTAs may start their prologue while
    // the previous kernel of the stream (normally the metadata kernel)
    // finishes; they read no input before griddepcontrol.wait.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kernel, kv_map, q_map, sc_map, prm);
    if (e != cudaSuccess) return cuda_fail(e, "mla_decode_kernel launch");
    return MLA_OK;
}

}  // namespace host
}  // namespace mla

// Scratch for callers that cannot allocate device memory: a fixed, file-scope
// device array that lives as long as the library is loaded.  Host code must not
// pass the array's name to a kernel (on the host it is only a stand-in); it
// passes the device address that cudaGetSymbolAddress returns for the current
// device.
static __device__ __align__(256) unsigned char g_static_workspace[MLA_STATIC_WORKSPACE_BYTES];

namespace mla {
namespace host {

std::mutex g_static_ws_mutex;
void *g_static_ws_ptr[64] = {nullptr};

// Device address of g_static_workspace on the current device, resolved once
// per device (the first call on a device does this; it makes no allocation).
mla_status_t static_workspace_address(void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= 64) return cuda_fail(cudaErrorInvalidDevice, "device index");
    std::lock_guard<std::mutex> lock(g_static_ws_mutex);
    if (!g_static_ws_ptr[dev]) {
        void *ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_static_workspace);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static workspace)");
        g_static_ws_ptr[dev] = ptr;
    }
    *out = g_static_ws_ptr[dev];
    return MLA_OK;
}

// Test hook for the bounded device waits (mla_debug_stall_cta): -1 = off.
std::atomic<int> g_debug_stall_cta{-1};

DecodeParams make_params(const int32_t *block_table, const int32_t *cache_seqlens, int B, int s_q, int H,
                         const Shape &sh, int64_t num_blocks, int max_blocks, float softmax_scale, int num_sms,
                         const int32_t *sched_meta, const int32_t *num_splits, void *workspace,
                         const WorkspaceLayout &wl, uint16_t *out, float *lse)
{
    DecodeParams prm;
    prm.block_table = block_table;
    prm.seqlens = cache_seqlens;
    prm.sched = sched_meta;
    prm.split_base = num_splits;
    prm.ws_o = static_cast<float *>(workspace);
    prm.ws_lse = reinterpret_cast<float *>(static_cast<char *>(workspace) + wl.lse_off);
    prm.out = out;
    prm.lse = lse;
    prm.err = const_cast<int32_t *>(sched_meta);
    prm.B = B;
    prm.s_q = s_q;
    prm.H = H;
    prm.G = sh.G;
    prm.num_sms = num_sms;
    prm.num_tuples = num_sms / sh.G;
    prm.max_blocks = max_blocks;
    prm.num_blocks = num_blocks;
    prm.scale_log2 = softmax_scale * 1.4426950408889634f;
    prm.ring = 0;
    prm.max_pieces = wl.pieces;
    prm.debug_stall_cta = g_debug_stall_cta.load(std::memory_order_relaxed);
    return prm;
}

}  // namespace host
}  // namespace mla

using namespace mla;
using namespace mla::host;

extern "C" mla_status_t mla_decode_combine(const int32_t *num_splits, const int32_t *sched_meta,
                                          const void *workspace, size_t workspace_bytes, int B, int s_q, int H,
                                          int num_sms, uint16_t *out, float *lse, void *stream);

namespace mla {
namespace host {

void clear_error() { g_last_error[0] = '\0'; }

// Checks shared by every decode entry point; `kv_align` is the cache
// pointer's alignment rule.
mla_status_t check_decode_args(const void *q, const void *kv, const void *kv_scale, bool fp8,
                               const int32_t *block_table, const int32_t *cache_seqlens, int B, int s_q, int H,
                               int64_t num_blocks, int max_blocks, float softmax_scale, int num_sms,
                               const int32_t *sched_meta, const int32_t *num_splits, const void *workspace,
                               size_t workspace_bytes, const uint16_t *out, const float *lse, Shape *sh,
                               WorkspaceLayout *wl)
{
    if (!q || !kv || (fp8 && !kv_scale) || !block_table || !cache_seqlens || !sched_meta || !num_splits ||
        !workspace || !out || !lse)
        return MLA_ERR_INVALID_ARG;
    if (B < 1 || B > kMaxBatch || num_blocks < 1 || num_blocks > INT32_MAX || max_blocks < 1)
        return MLA_ERR_INVALID_ARG;
    if (!std::isfinite(softmax_scale)) return MLA_ERR_INVALID_ARG;
    if (!resolve(s_q, H, sh)) return MLA_ERR_UNSUPPORTED_SHAPE;
    // FP8 cache: 16 or 32 query columns (H = 16 with s_q = 1 or 2, H = 32 with s_q = 1)
    if (fp8 && !(sh->G == 1 && (sh->N == 16 || (sh->N == 32 && s_q <= 2)))) return MLA_ERR_UNSUPPORTED_SHAPE;
    if (num_sms < sh->G || num_sms > kMaxSms) return MLA_ERR_UNSUPPORTED_SHAPE;
    if ((reinterpret_cast<uintptr_t>(q) & 15) || (reinterpret_cast<uintptr_t>(kv) & 15) ||
        (reinterpret_cast<uintptr_t>(kv_scale) & 15) || (reinterpret_cast<uintptr_t>(workspace) & 255) ||
        (reinterpret_cast<uintptr_t>(out) & 7) || (reinterpret_cast<uintptr_t>(lse) & 3) ||
        (reinterpret_cast<uintptr_t>(block_table) & 3) || (reinterpret_cast<uintptr_t>(cache_seqlens) & 3) ||
        (reinterpret_cast<uintptr_t>(sched_meta) & 3) || (reinterpret_cast<uintptr_t>(num_splits) & 3))
        return MLA_ERR_MISALIGNED;
    *wl = layout(B, s_q, *sh, num_sms);
    if (workspace_bytes < wl->total) return MLA_ERR_WORKSPACE_TOO_SMALL;
    if (static_cast<int64_t>(B) * s_q * H > INT32_MAX) return MLA_ERR_INVALID_ARG;
    return MLA_OK;
}

// q viewed as [B * s_q * H rows][576 cols]; box 64 cols x (heads per CTA) rows.
bool q_tensor_map(CUtensorMap *m, const uint16_t *q, int B, int s_q, int H, const Shape &sh)
{
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kDQK), static_cast<cuuint64_t>(B) * s_q * H};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kDQK) * 2};
    const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(sh.HG)};
    return tensor_map(m, "q", CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
}

mla_status_t decode_bf16(const uint16_t *q, const uint16_t *kv_cache, const int32_t *block_table,
                         const int32_t *cache_seqlens, int B, int s_q, int H, int64_t num_blocks, int max_blocks,
                         float softmax_scale, int num_sms, const int32_t *sched_meta, const int32_t *num_splits,
                         void *workspace, size_t workspace_bytes, uint16_t *out, float *lse, void *stream,
                         bool with_combine)
{
    clear_error();
    Shape sh;
    WorkspaceLayout wl;
    const mla_status_t chk = check_decode_args(q, kv_cache, nullptr, false, block_table, cache_seqlens, B, s_q, H,
                                               num_blocks, max_blocks, softmax_scale, num_sms, sched_meta,
                                               num_splits, workspace, workspace_bytes, out, lse, &sh, &wl);
    if (chk != MLA_OK) return chk;
    // kv_cache viewed as [num_blocks][64 rows][576 cols]; box 64 cols x 64 rows x 1 block.
    CUtensorMap kv_map, q_map;
    {
        const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kDQK), static_cast<cuuint64_t>(kPage),
                                    static_cast<cuuint64_t>(num_blocks)};
        const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kDQK) * 2, static_cast<cuuint64_t>(kPage) * kDQK * 2};
        const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(kPage), 1};
        if (!tensor_map(&kv_map, "kv", CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, kv_cache, dims, strides, box,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B))
            return MLA_ERR_CUDA;
    }
    if (!q_tensor_map(&q_map, q, B, s_q, H, sh)) return MLA_ERR_CUDA;

    const DecodeParams prm = make_params(block_table, cache_seqlens, B, s_q, H, sh, num_blocks, max_blocks,
                                         softmax_scale, num_sms, sched_meta, num_splits, workspace, wl, out, lse);
    const int grid = prm.num_tuples * sh.G;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // (the scale map is only read by the FP8 kernel; q_map stands in for it)
    mla_status_t rc;
    if (sh.N == 16) rc = launch_decode<16, 1, false>(kv_map, q_map, q_map, prm, grid, st);
    else if (sh.N == 32 && s_q == 1) rc = launch_decode<32, 1, false>(kv_map, q_map, q_map, prm, grid, st);
    else if (sh.N == 32) rc = launch_decode<32, 2, false>(kv_map, q_map, q_map, prm, grid, st);
    else if (s_q == 1) rc = launch_decode<64, 1, false>(kv_map, q_map, q_map, prm, grid, st);
    else if (s_q == 2) rc = launch_decode<64, 2, false>(kv_map, q_map, q_map, prm, grid, st);
    else if (s_q == 4) rc = launch_decode<64, 4, false>(kv_map, q_map, q_map, prm, grid, st);
    else rc = launch_decode<64, 8, false>(kv_map, q_map, q_map, prm, grid, st);
    if (rc != MLA_OK || !with_combine) return rc;
    return mla_decode_combine(num_splits, sched_meta, workspace, workspace_bytes, B, s_q, H, num_sms, out, lse,
                              stream);
}

mla_status_t decode_fp8(const uint16_t *q, const uint8_t *kv_codes, const float *kv_scale,
                        const int32_t *block_table, const int32_t *cache_seqlens, int B, int s_q, int H,
                        int64_t num_blocks, int max_blocks, float softmax_scale, int num_sms,
                        const int32_t *sched_meta, const int32_t *num_splits, void *workspace,
                        size_t workspace_bytes, uint16_t *out, float *lse, void *stream, bool with_combine)
{
    clear_error();
    Shape sh;
    WorkspaceLayout wl;
    const mla_status_t chk = check_decode_args(q, kv_codes, kv_scale, true, block_table, cache_seqlens, B, s_q, H,
                                               num_blocks, max_blocks, softmax_scale, num_sms, sched_meta,
                                               num_splits, workspace, workspace_bytes, out, lse, &sh, &wl);
    if (chk != MLA_OK) return chk;
    CUtensorMap kv_map, q_map, sc_map;
    // codes viewed as [num_blocks][64 rows][576 bytes]; box 128 bytes x 64 rows x 1 block, 128-byte
    // swizzled.  The rope group's box (columns 512..639) reads zeros past column 575.
    {
        const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kDQK), static_cast<cuuint64_t>(kPage),
                                    static_cast<cuuint64_t>(num_blocks)};
        const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kDQK), static_cast<cuuint64_t>(kPage) * kDQK};
        const cuuint32_t box[3] = {128, static_cast<cuuint32_t>(kPage), 1};
        if (!tensor_map(&kv_map, "kv fp8", CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, kv_codes, dims, strides, box,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B))
            return MLA_ERR_CUDA;
    }
    // token scales viewed as [num_blocks][64]; box 64 x 1 block (256 bytes)
    {
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kPage), static_cast<cuuint64_t>(num_blocks)};
        const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kPage) * 4};
        const cuuint32_t box[2] = {static_cast<cuuint32_t>(kPage), 1};
        if (!tensor_map(&sc_map, "kv scale", CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, kv_scale, dims, strides, box,
                        CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE))
            return MLA_ERR_CUDA;
    }
    if (!q_tensor_map(&q_map, q, B, s_q, H, sh)) return MLA_ERR_CUDA;
    const DecodeParams prm = make_params(block_table, cache_seqlens, B, s_q, H, sh, num_blocks, max_blocks,
                                         softmax_scale, num_sms, sched_meta, num_splits, workspace, wl, out, lse);
    const int grid = prm.num_tuples * sh.G;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    mla_status_t rc;
    if (sh.N == 16) rc = launch_decode<16, 1, true>(kv_map, q_map, sc_map, prm, grid, st);
    else if (s_q == 1) rc = launch_decode<32, 1, true>(kv_map, q_map, sc_map, prm, grid, st);
    else rc = launch_decode<32, 2, true>(kv_map, q_map, sc_map, prm, grid, st);
    if (rc != MLA_OK || !with_combine) return rc;
    return mla_decode_combine(num_splits, sched_meta, workspace, workspace_bytes, B, s_q, H, num_sms, out, lse,
                              stream);
}

}  // namespace host
}  // namespace mla

extern "C" {

size_t mla_sched_meta_ints(int num_sms)
{
    if (num_sms < 1 || num_sms > kMaxSms) return 0;
    return static_cast<size_t>(kSchedHeader) + static_cast<size_t>(kSchedEntry) * num_sms;
}

size_t mla_decode_workspace_size(int B, int s_q, int H, int num_sms)
{
    Shape sh;
    if (B < 1 || B > kMaxBatch || num_sms < 1 || num_sms > kMaxSms || !resolve(s_q, H, &sh) || num_sms < sh.G)
        return 0;
    return layout(B, s_q, sh, num_sms).total;
}

mla_status_t mla_decode_metadata(const int32_t *cache_seqlens, int B, int s_q, int H, int num_sms,
                                 int32_t *sched_meta, int32_t *num_splits, void *stream)
{
    clear_error();
    if (!cache_seqlens || !sched_meta || !num_splits) return MLA_ERR_INVALID_ARG;
    if (B < 1 || B > kMaxBatch) return MLA_ERR_INVALID_ARG;
    Shape sh;
    if (!resolve(s_q, H, &sh)) return MLA_ERR_UNSUPPORTED_SHAPE;
    if (num_sms < sh.G || num_sms > kMaxSms) return MLA_ERR_UNSUPPORTED_SHAPE;
    if ((reinterpret_cast<uintptr_t>(cache_seqlens) | reinterpret_cast<uintptr_t>(sched_meta) |
         reinterpret_cast<uintptr_t>(num_splits)) & 3)
        return MLA_ERR_MISALIGNED;
    const int tuples = num_sms / sh.G;
    const size_t smem = B <= 32 ? 32 * sizeof(int) : (2 * static_cast<size_t>(B + 1) + 33) * sizeof(int);
    mla_metadata_kernel<<<1, kMetaThreads, smem, static_cast<cudaStream_t>(stream)>>>(
        cache_seqlens, B, s_q, H, num_sms, tuples, sh.G, sched_meta, num_splits);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "mla_metadata_kernel launch");
    return MLA_OK;
}

mla_status_t mla_decode_combine(const int32_t *num_splits, const int32_t *sched_meta, const void *workspace,
                                size_t workspace_bytes, int B, int s_q, int H, int num_sms, uint16_t *out,
                                float *lse, void *stream)
{
    clear_error();
    if (!num_splits || !sched_meta || !workspace || !out || !lse) return MLA_ERR_INVALID_ARG;
    if (B < 1 || B > kMaxBatch) return MLA_ERR_INVALID_ARG;
    Shape sh;
    if (!resolve(s_q, H, &sh)) return MLA_ERR_UNSUPPORTED_SHAPE;
    if (num_sms < sh.G || num_sms > kMaxSms) return MLA_ERR_UNSUPPORTED_SHAPE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255) || (reinterpret_cast<uintptr_t>(out) & 7) ||
        (reinterpret_cast<uintptr_t>(lse) & 3) || (reinterpret_cast<uintptr_t>(num_splits) & 3) ||
        (reinterpret_cast<uintptr_t>(sched_meta) & 3))
        return MLA_ERR_MISALIGNED;
    const WorkspaceLayout wl = layout(B, s_q, sh, num_sms);
    if (workspace_bytes < wl.total) return MLA_ERR_WORKSPACE_TOO_SMALL;
    const float *ws_o = static_cast<const float *>(workspace);
    const float *ws_lse = reinterpret_cast<const float *>(static_cast<const char *>(workspace) + wl.lse_off);
    const int64_t rows = static_cast<int64_t>(B) * s_q * H;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(rows));
    cfg.blockDim = dim3(kCombineThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // one wave of 4 blocks per SM (of num_sms SMs): the wide batch
    const bool wide = rows <= 4ll * num_sms;
    cudaError_t e = cudaLaunchKernelEx(&cfg, wide ? mla_combine_kernel<20> : mla_combine_kernel<8>, num_splits, ws_o,
                                       ws_lse, B, s_q, H, sh.HG, sh.G,
                                       wl.pieces, out, lse, const_cast<int32_t *>(sched_meta));
    if (e != cudaSuccess) return cuda_fail(e, "mla_combine_kernel launch");
    return MLA_OK;
}

mla_status_t mla_decode_attention(const uint16_t *q, const uint16_t *kv_cache, const int32_t *block_table,
                                  const int32_t *cache_seqlens, int B, int s_q, int H, int64_t num_blocks,
                                  int max_blocks, float softmax_scale, int num_sms, const int32_t *sched_meta,
                                  const int32_t *num_splits, void *workspace, size_t workspace_bytes, uint16_t *out,
                                  float *lse, void *stream)
{
    return decode_bf16(q, kv_cache, block_table, cache_seqlens, B, s_q, H, num_blocks, max_blocks, softmax_scale,
                       num_sms, sched_meta, num_splits, workspace, workspace_bytes, out, lse, stream, false);
}

mla_status_t mla_decode(const uint16_t *q, const uint16_t *kv_cache, const int32_t *block_table,
                        const int32_t *cache_seqlens, int B, int s_q, int H, int64_t num_blocks, int max_blocks,
                        float softmax_scale, int num_sms, const int32_t *sched_meta, const int32_t *num_splits,
                        void *workspace, size_t workspace_bytes, uint16_t *out, float *lse, void *stream)
{
    return decode_bf16(q, kv_cache, block_table, cache_seqlens, B, s_q, H, num_blocks, max_blocks, softmax_scale,
                       num_sms, sched_meta, num_splits, workspace, workspace_bytes, out, lse, stream, true);
}

mla_status_t mla_decode_attention_fp8(const uint16_t *q, const uint8_t *kv_codes, const float *kv_scale,
                                      const int32_t *block_table, const int32_t *cache_seqlens, int B, int s_q,
                                      int H, int64_t num_blocks, int max_blocks, float softmax_scale, int num_sms,
                                      const int32_t *sched_meta, const int32_t *num_splits, void *workspace,
                                      size_t workspace_bytes, uint16_t *out, float *lse, void *stream)
{
    return decode_fp8(q, kv_codes, kv_scale, block_table, cache_seqlens, B, s_q, H, num_blocks, max_blocks,
                      softmax_scale, num_sms, sched_meta, num_splits, workspace, workspace_bytes, out, lse, stream,
                      false);
}

mla_status_t mla_decode_fp8(const uint16_t *q, const uint8_t *kv_codes, const float *kv_scale,
                            const int32_t *block_table, const int32_t *cache_seqlens, int B, int s_q, int H,
                            int64_t num_blocks, int max_blocks, float softmax_scale, int num_sms,
                            const int32_t *sched_meta, const int32_t *num_splits, void *workspace,
                            size_t workspace_bytes, uint16_t *out, float *lse, void *stream)
{
    return decode_fp8(q, kv_codes, kv_scale, block_table, cache_seqlens, B, s_q, H, num_blocks, max_blocks,
                      softmax_scale, num_sms, sched_meta, num_splits, workspace, workspace_bytes, out, lse, stream,
                      true);
}

mla_status_t mla_decode_static_workspace(const uint16_t *q, const uint16_t *kv_cache, const int32_t *block_table,
                                         const int32_t *cache_seqlens, int B, int s_q, int H, int64_t num_blocks,
                                         int max_blocks, float softmax_scale, int num_sms,
                                         const int32_t *sched_meta, const int32_t *num_splits, uint16_t *out,
                                         float *lse, void *stream)
{
    clear_error();
    const size_t need = mla_decode_workspace_size(B, s_q, H, num_sms);
    if (need == 0) {
        if (B < 1 || B > kMaxBatch) return MLA_ERR_INVALID_ARG;
        return MLA_ERR_UNSUPPORTED_SHAPE;
    }
    if (need > MLA_STATIC_WORKSPACE_BYTES) {
        snprintf(g_last_error, sizeof g_last_error,
                 "mla_decode_static_workspace: this shape needs %zu bytes of workspace, the built-in one holds %zu",
                 need, static_cast<size_t>(MLA_STATIC_WORKSPACE_BYTES));
        return MLA_ERR_WORKSPACE_TOO_SMALL;
    }
    void *ws = nullptr;
    const mla_status_t rc = static_workspace_address(&ws);
    if (rc != MLA_OK) return rc;
    return mla_decode(q, kv_cache, block_table, cache_seqlens, B, s_q, H, num_blocks, max_blocks, softmax_scale,
                      num_sms, sched_meta, num_splits, ws, MLA_STATIC_WORKSPACE_BYTES, out, lse, stream);
}

void mla_debug_stall_cta(int cta) { g_debug_stall_cta.store(cta < 0 ? -1 : cta, std::memory_order_relaxed); }

mla_status_t mla_get_device_error(const int32_t *sched_meta, int32_t *host_code, void *stream)
{
    clear_error();
    if (!sched_meta || !host_code) return MLA_ERR_INVALID_ARG;
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    e = cudaMemcpy(host_code, sched_meta, sizeof(int32_t), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(error word)");
    return *host_code ? MLA_ERR_DEVICE_CHECK : MLA_OK;
}

const char *mla_status_string(mla_status_t status)
{
    switch (status) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG";
    case MLA_ERR_MISALIGNED: return "MLA_ERR_MISALIGNED";
    case MLA_ERR_UNSUPPORTED_SHAPE: return "MLA_ERR_UNSUPPORTED_SHAPE";
    case MLA_ERR_WORKSPACE_TOO_SMALL: return "MLA_ERR_WORKSPACE_TOO_SMALL";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
    case MLA_ERR_DEVICE_CHECK: return "MLA_ERR_DEVICE_CHECK";
    }
    return "MLA_ERR_UNKNOWN";
}

const char *mla_last_error_message(void) { return g_last_error; }

}  // extern "C"
