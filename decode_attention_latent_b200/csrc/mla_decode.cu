// mla_decode.cu -- absorbed-form MLA decode for B200 (sm_100a).
//
// Three kernels behind the C ABI of include/mla_decode.h:
//
//   mla_metadata_kernel  split-KV schedule: the 128-token tiles of all
//                        sequences are laid end to end and cut into equal
//                        contiguous ranges, one per CTA group.
//   mla_decode_*_kernel  one persistent CTA per SM.  Per 128-token tile:
//                          TMA gathers the tile's two pages through the page
//                          table into a ring of 16 KB shared-memory slots
//                          (one slot = 64 columns of 128 rows, 128-byte
//                          swizzled);
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
// Two variants of the attention kernel:
//
//   tv (N <= 32)  The V part of each tile is copied, transposed, from its
//                 shared-memory slots into TMEM by four transposer warps as
//                 soon as it lands (ldmatrix.trans -> tcgen05.st), and the
//                 output MMA reads A = V^T from TMEM.  A slot is released once
//                 the score MMA and the transposer have read it, so the ring
//                 never waits on the softmax.  Warps: producer, score MMA,
//                 4 softmax, 4 transposer, output MMA.
//   ss (N = 64)   TMEM cannot hold O^T, S^T and a tile of V^T at N = 64, so
//                 the tile stays in shared memory until the output MMA reads
//                 V^T from it (MN-major A); the softmax writes P^T into the
//                 dead rope slot.  Warps: producer, MMA, 4 softmax.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <climits>
#include <mutex>

#include "../../include/mla_decode.h"
#include "sm100_ptx.cuh"

namespace mla {

constexpr int kDQK = MLA_D_QK;
constexpr int kDV = MLA_D_V;
constexpr int kPage = MLA_PAGE;
constexpr int kTile = MLA_TILE;
constexpr int kChunks = kDQK / 64;              // 9 column chunks per row
constexpr uint32_t kSlotBytes = 16384;          // 128 rows x 128 B
constexpr uint32_t kPageChunkBytes = 8192;      // 64 rows x 128 B
constexpr int kThreadsSS = 192;                 // producer, MMA, 4 softmax warps
constexpr int kThreadsTV = 352;                 // + 4 transposer warps, output-MMA warp
constexpr int kMaxRing = 16;
constexpr int kMinRing = 9;                     // a whole tile must fit: its slots are released per tile
constexpr int kMaxBatch = 4096;
constexpr int kMaxSms = 4096;
constexpr int kSchedHeader = 16;
constexpr int kSchedEntry = 8;
constexpr int kSchedMagic = 0x4D4C4144;         // "MLAD"
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // bounded device waits: 2 s
constexpr float kLn2 = 0.6931471805599453f;
constexpr uint32_t kVtCol = 256;                // tv: V^T occupies TMEM columns [256, 512)

// Barrier indices inside the "misc" shared-memory region.
constexpr int kBarFull = 0;                   // [kMaxRing]
constexpr int kBarEmpty = kMaxRing;           // [kMaxRing]
constexpr int kBarQFull = 2 * kMaxRing;
constexpr int kBarQEmpty = 2 * kMaxRing + 1;
constexpr int kBarSFull = 2 * kMaxRing + 2;   // [2]: one per S^T buffer
constexpr int kBarSEmpty = 2 * kMaxRing + 4;  // [2] (tv)
constexpr int kBarPFull = 2 * kMaxRing + 6;
constexpr int kBarODone = 2 * kMaxRing + 7;
constexpr int kBarVtFull = 2 * kMaxRing + 8;  // (tv)
constexpr int kBarDrain = 2 * kMaxRing + 9;
constexpr int kBarDrainO = 2 * kMaxRing + 10; // (tv)
constexpr int kNumBars = 2 * kMaxRing + 11;
// The reduction buffers after the barriers are read as float4: keep them
// 16-byte aligned (rounded to 128 B).
constexpr uint32_t kMiscRedOffset = (kNumBars * 8 + 127) / 128 * 128;
static_assert(kMiscRedOffset % 16 == 0, "reduction buffers must be 16-byte aligned");

template <int N>
constexpr uint32_t misc_bytes()
{
    // barriers, max-reduction buffer [2][4][N], sum buffer [4][N], tmem holder, abort flag
    return kMiscRedOffset + (2 * 4 * N + 4 * N) * 4 + 16;
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

__global__ void __launch_bounds__(kMetaThreads, 1)
mla_metadata_kernel(const int32_t *__restrict__ seqlens, int B, int s_q, int H, int num_sms,
                    int num_tuples, int G, int32_t *__restrict__ sched, int32_t *__restrict__ split_base)
{
    __shared__ int prefix[kMaxBatch + 1];
    __shared__ int nsplit[kMaxBatch + 1];
    __shared__ int warp_sums[32];
    __shared__ int bad_len;
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
        int32_t *e = sched + kSchedHeader + k * kSchedEntry;
        const int start = k * per;
        if (start >= total) {
            e[0] = -1; e[1] = 0; e[2] = -1; e[3] = 0; e[4] = 0; e[5] = 0; e[6] = 0; e[7] = 0;
            continue;
        }
        const int end = min(start + per, total);
        const int b0 = last_at_or_below(prefix, B, start);
        const int b1 = last_at_or_below(prefix, B, end - 1);
        e[0] = b0;
        e[1] = start - prefix[b0];
        e[2] = b1;
        e[3] = end - prefix[b1];
        e[4] = k - prefix[b0] / per;  // index of this group's piece of sequence b0
        e[5] = 0; e[6] = 0; e[7] = 0;
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
        sched[0] = bad_len ? MLA_DEVERR_SEQLEN : 0;
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
}

// All lanes of the calling warp wait; the outcome is agreed warp-wide so the
// warp stays converged even when a bounded wait runs out in some lanes only.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag, int32_t *err,
                                          bool honour_abort = true)
{
    const bool ok = wait_bounded(bar, parity, abort_flag, err, honour_abort);
    return __all_sync(0xffffffffu, ok);
}

// Page-table window: lane j returns the physical block of page `first + j`
// (0 for pages outside [0, npages), and, with an error bit, for entries that
// do not name a block of the cache).
__device__ __forceinline__ int load_pages(const int32_t *bt, int first, int npages, const DecodeParams &p, int lane)
{
    const int idx = first + lane;
    int id = 0;
    if (idx < npages) {
        if (idx >= p.max_blocks) {
            atomicOr(p.err, MLA_DEVERR_SEQLEN);
        } else {
            id = __ldg(bt + idx);
            if (id < 0 || static_cast<int64_t>(id) >= p.num_blocks) {
                atomicOr(p.err, MLA_DEVERR_BLOCK_TABLE);
                id = 0;
            }
        }
    }
    return id;
}

// ================================================================ decode
template <int N, int SQ>
struct Cfg {
    static constexpr bool TV = N <= 32;                    // variant (see the file header)
    static constexpr int HG = N / SQ;                      // heads per CTA
    static constexpr int NCH = N / 16;                     // 16-column TMEM chunks
    static constexpr uint32_t QCHUNK = N * 128u;           // bytes: 64 columns of N rows
    static constexpr uint32_t QBYTES = kChunks * QCHUNK;   // N x 576 bf16
    static constexpr uint32_t PBYTES = TV ? 2 * 2 * QCHUNK : 0;  // tv: 2 P^T buffers of N x 128 bf16
    static constexpr uint32_t S_COL = 4 * N;               // S^T buffers after the 4 O^T blocks
    static constexpr uint32_t TMEM_COLS = TV ? 512u : ((5 * N <= 256) ? 256u : 512u);
    static constexpr int THREADS = TV ? kThreadsTV : kThreadsSS;
    static_assert(!TV || 6 * N <= static_cast<int>(kVtCol), "O^T and S^T must fit below V^T");
};

struct Smem {
    uint32_t ring, q, p;     // shared-window addresses: slot ring, Q, P^T buffers (tv)
    uint32_t bars;           // address of barrier 0
    float *red, *lred;
    uint32_t *tmem_holder;
    volatile int *abort_flag;
    __device__ __forceinline__ uint32_t bar(int i) const { return bars + 8u * i; }
    __device__ __forceinline__ uint32_t slot(int s) const { return ring + kSlotBytes * s; }
};

// Output of one range: reduce the per-row sums across the four softmax warps,
// normalise O^T and write either the final out/lse or the fp32 piece for the
// combine kernel.  O^T must be complete (and fenced) when this is called.
template <int N, int SQ>
__device__ void range_epilogue(const DecodeParams &p, const Smem &sm, uint32_t tmem, int b, int split, int g,
                               const float (&m)[N], float (&l)[N])
{
    using C = Cfg<N, SQ>;
    constexpr int HG = C::HG;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const int tid = threadIdx.x - 64;
    const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
#pragma unroll
    for (int n = 0; n < N; ++n) {
        const float s = warp_sum(l[n]);
        if (lane == 0) sm.lred[wq * N + n] = s;
    }
    __syncwarp();
    ptx::named_bar_sync(1, 128);
#pragma unroll
    for (int n = 0; n < N; ++n)
        l[n] = (sm.lred[n] + sm.lred[N + n]) + (sm.lred[2 * N + n] + sm.lred[3 * N + n]);

    const int nsplit = p.split_base[b + 1] - p.split_base[b];
    const bool final_out = nsplit <= 1;
    int piece = (p.split_base[b] + split) * p.G + g;
    bool write_ok = true;
    if (!final_out && (piece < 0 || piece >= p.max_pieces)) {
        if (tid == 0) atomicOr(p.err, MLA_DEVERR_SCHEDULE);
        write_ok = false;
        piece = 0;
    }
#pragma unroll 1
    for (int j = 0; j < 4; ++j) {
        const int dim = j * 128 + row;
#pragma unroll
        for (int ch = 0; ch < C::NCH; ++ch) {
            float v[16];
            ptx::tmem_ld16(tmem + lane_base + j * N + ch * 16, v);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int n = ch * 16 + e;
                const int i = n / HG, hl = n % HG;
                const float val = l[n] > 0.f ? v[e] / l[n] : 0.f;
                if (final_out) {
                    const int64_t o = ((static_cast<int64_t>(b) * SQ + i) * p.H + g * HG + hl) * kDV + dim;
                    p.out[o] = __bfloat16_as_ushort(__float2bfloat16_rn(val));
                } else if (write_ok) {
                    const int64_t o = ((static_cast<int64_t>(piece) * SQ + i) * HG + hl) * kDV + dim;
                    p.ws_o[o] = val;
                }
            }
        }
    }
#pragma unroll
    for (int n = 0; n < N; ++n) {
        if (tid == n) {
            const int i = n / HG, hl = n % HG;
            const float val = l[n] > 0.f ? (m[n] + log2f(l[n])) * kLn2 : -INFINITY;
            if (final_out)
                p.lse[(static_cast<int64_t>(b) * SQ + i) * p.H + g * HG + hl] = val;
            else if (write_ok)
                p.ws_lse[(static_cast<int64_t>(piece) * SQ + i) * HG + hl] = val;
        }
    }
    __syncwarp();
    ptx::tc_fence_before();
}

// Max over the 32 lanes of a warp for 16 columns at once: halving exchanges
// (16 shuffles in all).  Returns, in lane l, the maximum of column l >> 1.
__device__ __forceinline__ float warp_colmax16(float (&x)[16], int lane)
{
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const bool hi = lane & 16;
        const float send = hi ? x[j] : x[j + 8];
        const float keep = hi ? x[j + 8] : x[j];
        x[j] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, 16));
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const bool hi = lane & 8;
        const float send = hi ? x[j] : x[j + 4];
        const float keep = hi ? x[j + 4] : x[j];
        x[j] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, 8));
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const bool hi = lane & 4;
        const float send = hi ? x[j] : x[j + 2];
        const float keep = hi ? x[j + 2] : x[j];
        x[j] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, 4));
    }
    {
        const bool hi = lane & 2;
        const float send = hi ? x[0] : x[1];
        const float keep = hi ? x[1] : x[0];
        x[0] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, 2));
    }
    return fmaxf(x[0], __shfl_xor_sync(0xffffffffu, x[0], 1));
}

// ====================================================== ss variant (N = 64)
// A tile occupies 9 consecutive ring slots starting at s0.  The four
// (even, odd) V chunk pairs must sit in adjacent slots (an M = 128 block of
// V^T spans both), so when the window wraps past the ring's last slot the
// rope chunk is placed first or last to keep the wrap between two pairs.
__device__ __forceinline__ bool rope_first_at(uint32_t s0, int R)
{
    if (static_cast<int>(s0) + 8 < R) return false;
    const int w = R - 1 - static_cast<int>(s0);
    return (w & 1) == 0;
}

__device__ __forceinline__ int pos_of_chunk(int c, bool rope_first)
{
    return rope_first ? (c == kChunks - 1 ? 0 : c + 1) : c;
}

// -- ss producer warp: issues every TMA load --------------------------------
template <int N, int SQ>
__device__ void ss_producer(const DecodeParams &p, const Range &w, int g, const Smem &sm,
                             const CUtensorMap *kv_map, const CUtensorMap *q_map)
{
    using C = Cfg<N, SQ>;
    const int lane = threadIdx.x & 31;
    const int R = p.ring;
    uint32_t cc = 0;  // chunk-slot uses so far
    int qi = 0;       // Q loads so far
    bool ok = true;
    for (int b = w.b0; b <= w.b1 && ok; ++b) {
        const int L = max(0, __ldg(p.seqlens + b));
        const int nt = tiles_of(L);
        const int tb = (b == w.b0) ? w.t0 : 0;
        const int te = min((b == w.b1) ? w.t1 : nt, nt);
        if (tb >= te) continue;
        const int32_t *bt = p.block_table + static_cast<int64_t>(b) * p.max_blocks;
        const int npages = (L + kPage - 1) / kPage;
        int win = 2 * tb;
        int cur = load_pages(bt, win, npages, p, lane);
        int nxt = load_pages(bt, win + 32, npages, p, lane);

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
            const uint32_t bytes = live1 ? 2 * kPageChunkBytes : kPageChunkBytes;
            const uint32_t s0 = cc % R;
            const bool rf = rope_first_at(s0, R);
#pragma unroll 1
            for (int k = 0; k < kChunks; ++k) {
                const int chunk = rf ? (k == 0 ? kChunks - 1 : k - 1) : k;
                const uint32_t u = cc + k;
                const int slot = static_cast<int>(u % R);
                if (!warp_wait(sm.bar(kBarEmpty + slot), ((u / R) & 1) ^ 1, sm.abort_flag, p.err)) {
                    ok = false;
                    cc += k;  // uses issued so far in this tile
                    break;
                }
                ptx::mbar_arrive_expect_tx_elect(sm.bar(kBarFull + slot), bytes);
                ptx::tma_load_3d_elect(sm.slot(slot), kv_map, sm.bar(kBarFull + slot), chunk * 64, 0, phys0);
                if (live1)
                    ptx::tma_load_3d_elect(sm.slot(slot) + kPageChunkBytes, kv_map, sm.bar(kBarFull + slot),
                                           chunk * 64, 0, phys1);
            }
            if (ok) cc += kChunks;
        }
    }
    if (!ok) {
        // Let every load this warp issued land before the CTA exits.
        const uint32_t first = cc > static_cast<uint32_t>(R) ? cc - R : 0;
        for (uint32_t u = first; u < cc; ++u)
            warp_wait(sm.bar(kBarFull + static_cast<int>(u % R)), (u / R) & 1, sm.abort_flag, p.err, false);
    }
}

// -- ss MMA warp: issues every tcgen05.mma -----------------------------------
template <int N, int SQ>
__device__ void ss_mma(const DecodeParams &p, const Range &w, const Smem &sm, uint32_t tmem)
{
    using C = Cfg<N, SQ>;
    constexpr uint32_t idS = ptx::idesc_bf16_f32(128, N, false, false);  // K (cache) K-major, Q K-major
    constexpr uint32_t idO = ptx::idesc_bf16_f32(128, N, true, false);   // V^T MN-major, P^T K-major
    const int R = p.ring;
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
        for (int t = tb; t < te; ++t) {
            const uint32_t s0 = cc % R;
            const bool rf = rope_first_at(s0, R);
            // S^T[128 tokens x N] = K[128 x 576] . Q^T[576 x N], chunk by chunk
#pragma unroll 1
            for (int c = 0; c < kChunks; ++c) {
                const uint32_t u = cc + pos_of_chunk(c, rf);
                const int slot = static_cast<int>(u % R);
                if (!(ok = warp_wait(sm.bar(kBarFull + slot), (u / R) & 1, sm.abort_flag, p.err))) break;
                ptx::tc_fence_after();
                const uint32_t a0 = sm.slot(slot);
                const uint32_t b0 = sm.q + c * C::QCHUNK;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    ptx::mma_bf16_ss_elect(tmem + C::S_COL, ptx::desc_sw128(a0 + 32u * k, 16, 1024),
                                           ptx::desc_sw128(b0 + 32u * k, 16, 1024), idS, (c | k) != 0);
            }
            if (!ok) break;
            ptx::mma_commit_elect(sm.bar(kBarSFull));
            if (t == te - 1) ptx::mma_commit_elect(sm.bar(kBarQEmpty));
            // O^T[512 x N] += V^T[512 x 128 tokens] . P^T[128 x N]
            if (!(ok = warp_wait(sm.bar(kBarPFull), it & 1, sm.abort_flag, p.err))) break;
            ptx::tc_fence_after();
            const int rope_slot = static_cast<int>((s0 + pos_of_chunk(kChunks - 1, rf)) % R);
            const uint32_t pa = sm.slot(rope_slot);
#pragma unroll 1
            for (int j = 0; j < 4; ++j) {
                const int vslot = static_cast<int>((s0 + pos_of_chunk(2 * j, rf)) % R);
                const uint32_t va = sm.slot(vslot);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    ptx::mma_bf16_ss_elect(tmem + j * N, ptx::desc_sw128(va + 2048u * kk, kSlotBytes, 1024),
                                           ptx::desc_sw128(pa + (kk >> 2) * C::QCHUNK + 32u * (kk & 3), 16, 1024),
                                           idO, (t != tb) || (kk != 0));
                ptx::mma_commit_elect(sm.bar(kBarEmpty + vslot));
                ptx::mma_commit_elect(sm.bar(kBarEmpty + (vslot + 1) % R));
            }
            ptx::mma_commit_elect(sm.bar(kBarEmpty + rope_slot));
            ptx::mma_commit_elect(sm.bar(kBarODone));
            cc += kChunks;
            ++it;
        }
    }
    // Every MMA this warp issued must finish before TMEM is released.
    ptx::mma_commit_elect(sm.bar(kBarDrain));
    warp_wait(sm.bar(kBarDrain), 0, sm.abort_flag, p.err, false);
}

// -- ss softmax / epilogue: 4 warps, thread = one TMEM lane = one token row ---
template <int N, int SQ>
__device__ void ss_softmax(const DecodeParams &p, const Range &w, int g, const Smem &sm, uint32_t tmem)
{
    using C = Cfg<N, SQ>;
    constexpr int HG = C::HG;
    constexpr int NCH = C::NCH;
    constexpr bool kKeepScores = NCH <= 2;  // keep S in registers between the passes
    const int R = p.ring;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wq = warp & 3;              // TMEM lane quadrant this warp may access
    const int row = wq * 32 + lane;       // token row within the tile
    const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
    const float NEG_INF = -INFINITY;
    uint32_t cc = 0, it = 0;
    bool ok = true;

    for (int b = w.b0; b <= w.b1 && ok; ++b) {
        const int L = max(0, __ldg(p.seqlens + b));
        const int nt = tiles_of(L);
        const int tb = (b == w.b0) ? w.t0 : 0;
        const int te = min((b == w.b1) ? w.t1 : nt, nt);
        if (tb >= te) continue;
        const int split = (b == w.b0) ? w.split0 : 0;
        const int nvis0 = max(0, L - SQ + 1);  // tokens visible to query position 0
        float m[N], l[N];
#pragma unroll
        for (int n = 0; n < N; ++n) { m[n] = NEG_INF; l[n] = 0.f; }

        for (int t = tb; t < te; ++t) {
            const uint32_t s0 = cc % R;
            const bool rf = rope_first_at(s0, R);
            const bool got_s = wait_bounded(sm.bar(kBarSFull), it & 1, sm.abort_flag, p.err);
            __syncwarp();
            ok = ptx::named_bar_and(1, 128, got_s);
            if (!ok) break;
            ptx::tc_fence_after();
            const int tok = t * kTile + row;
            const bool vis0 = tok < nvis0, vis1 = tok < L;
            float *red = sm.red + (it & 1) * 4 * N;
            // pass 1: masked log2-domain scores and their per-column maximum
            float sc[kKeepScores ? NCH : 1][16];
#pragma unroll
            for (int ch = 0; ch < NCH; ++ch) {
                float v[16];
                ptx::tmem_ld16(tmem + lane_base + C::S_COL + ch * 16, v);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int n = ch * 16 + e;
                    const bool vis = (SQ == 2 && n >= HG) ? vis1 : vis0;
                    v[e] = vis ? v[e] * p.scale_log2 : NEG_INF;
                    if (kKeepScores) sc[kKeepScores ? ch : 0][e] = v[e];
                }
                const float cmax = warp_colmax16(v, lane);
                if ((lane & 1) == 0) red[wq * N + ch * 16 + (lane >> 1)] = cmax;
            }
            __syncwarp();
            ptx::named_bar_sync(1, 128);
            // pass 2: running max, weights, P^T into the rope slot, running sums
            const int rope_slot = static_cast<int>((s0 + pos_of_chunk(kChunks - 1, rf)) % R);
            const uint32_t pa = sm.slot(rope_slot) + (row >> 6) * C::QCHUNK;
            const uint32_t pcol = static_cast<uint32_t>(row & 63);
            bool any_rescale = false;
            float alpha[N];
#pragma unroll
            for (int ch = 0; ch < NCH; ++ch) {
                float v[16];
                if (kKeepScores) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) v[e] = sc[kKeepScores ? ch : 0][e];
                } else {
                    ptx::tmem_ld16(tmem + lane_base + C::S_COL + ch * 16, v);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int n = ch * 16 + e;
                        const bool vis = (SQ == 2 && n >= HG) ? vis1 : vis0;
                        v[e] = vis ? v[e] * p.scale_log2 : NEG_INF;
                    }
                }
                float tmax[16];
                {
                    const float4 *r4 = reinterpret_cast<const float4 *>(red + ch * 16);
#pragma unroll
                    for (int e4 = 0; e4 < 4; ++e4) {
                        const float4 a0 = r4[e4], a1 = r4[N / 4 + e4], a2 = r4[2 * (N / 4) + e4],
                                     a3 = r4[3 * (N / 4) + e4];
                        tmax[4 * e4 + 0] = fmaxf(fmaxf(a0.x, a1.x), fmaxf(a2.x, a3.x));
                        tmax[4 * e4 + 1] = fmaxf(fmaxf(a0.y, a1.y), fmaxf(a2.y, a3.y));
                        tmax[4 * e4 + 2] = fmaxf(fmaxf(a0.z, a1.z), fmaxf(a2.z, a3.z));
                        tmax[4 * e4 + 3] = fmaxf(fmaxf(a0.w, a1.w), fmaxf(a2.w, a3.w));
                    }
                }
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int n = ch * 16 + e;
                    const float mnew = fmaxf(m[n], tmax[e]);
                    // The reference max follows the true running max, so the
                    // largest weight of a range is exactly 1.
                    const bool need = mnew > m[n];
                    alpha[n] = need ? ptx::ex2_approx(m[n] - mnew) : 1.f;
                    if (need) {
                        m[n] = mnew;
                        any_rescale = true;
                    }
                    const float mu = (m[n] == NEG_INF) ? 0.f : m[n];
                    const float pr = ptx::ex2_approx(v[e] - mu);  // masked entries: 2^-inf = 0
                    l[n] = l[n] * alpha[n] + pr;
                    const uint32_t addr = pa + n * 128u + ((((pcol >> 3) ^ static_cast<uint32_t>(n & 7)) << 4)) +
                                          ((pcol & 7u) << 1);
                    ptx::st_shared_b16(addr, __bfloat16_as_ushort(__float2bfloat16_rn(pr)));
                }
            }
            // rows past the end of the sequence: make their V bytes zero so
            // that P = 0 meets finite values in the output MMA
            if (tok >= L) {
#pragma unroll 1
                for (int c = 0; c < kChunks - 1; ++c) {
                    const int vs = static_cast<int>((s0 + pos_of_chunk(c, rf)) % R);
                    const uint32_t ra = sm.slot(vs) + row * 128u;
#pragma unroll
                    for (int q16 = 0; q16 < 8; ++q16) ptx::st_shared_zero16(ra + q16 * 16u);
                }
            }
            __syncwarp();
            // rescale the O^T columns whose reference max moved (not needed
            // on the first tile of a range: its output MMA overwrites O^T)
            if (any_rescale && t != tb) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
#pragma unroll
                    for (int ch = 0; ch < NCH; ++ch) {
                        float v[16];
                        const uint32_t ta = tmem + lane_base + j * N + ch * 16;
                        ptx::tmem_ld16(ta, v);
                        ptx::tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] *= alpha[ch * 16 + e];
                        ptx::tmem_st16(ta, v);
                    }
                }
                ptx::tmem_wait_st();
            }
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            ptx::mbar_arrive(sm.bar(kBarPFull));
            cc += kChunks;
            ++it;
        }
        if (!ok) break;

        // ---- epilogue of this range
        const bool got_o = wait_bounded(sm.bar(kBarODone), (it - 1) & 1, sm.abort_flag, p.err);
        __syncwarp();
        ok = ptx::named_bar_and(1, 128, got_o);
        if (!ok) break;
        ptx::tc_fence_after();
        range_epilogue<N, SQ>(p, sm, tmem, b, split, g, m, l);
    }
}

// ====================================================== tv variant (N <= 32)
// K position, in the output MMA, of token r of a tile.  ldmatrix.trans hands
// each thread token pairs (2q, 2q+1) and (8+2q, 9+2q) of a 16-token group for
// one latent dim; stored as TMEM columns 2q and 2q+1 of that dim's lane they
// give the order 0,1,8,9,2,3,10,11,4,5,12,13,6,7,14,15 within each group.
// P^T is written in the same order, so the contraction is unchanged.
__device__ __forceinline__ int tv_kpos(int r)
{
    const int g = r & ~15, rr = r & 15;
    return g + (rr < 8 ? 2 * (rr & ~1) + (rr & 1) : 2 * ((rr - 8) & ~1) + 2 + (rr & 1));
}

// -- tv producer warp: Q per range, then each tile's 9 chunks in order ----
template <int N, int SQ>
__device__ void tv_producer(const DecodeParams &p, const Range &w, int g, const Smem &sm,
                            const CUtensorMap *kv_map, const CUtensorMap *q_map)
{
    using C = Cfg<N, SQ>;
    const int lane = threadIdx.x & 31;
    const uint32_t R = static_cast<uint32_t>(p.ring);
    uint32_t cc = 0;  // chunk-slot uses so far
    int qi = 0;       // Q loads so far
    bool ok = true;
    for (int b = w.b0; b <= w.b1 && ok; ++b) {
        const int L = max(0, __ldg(p.seqlens + b));
        const int nt = tiles_of(L);
        const int tb = (b == w.b0) ? w.t0 : 0;
        const int te = min((b == w.b1) ? w.t1 : nt, nt);
        if (tb >= te) continue;
        const int32_t *bt = p.block_table + static_cast<int64_t>(b) * p.max_blocks;
        const int npages = (L + kPage - 1) / kPage;
        int win = 2 * tb;
        int cur = load_pages(bt, win, npages, p, lane);
        int nxt = load_pages(bt, win + 32, npages, p, lane);

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
            const uint32_t bytes = live1 ? 2 * kPageChunkBytes : kPageChunkBytes;
#pragma unroll 1
            for (int c = 0; c < kChunks; ++c) {
                const uint32_t u = cc + c;
                const int slot = static_cast<int>(u % R);
                if (!warp_wait(sm.bar(kBarEmpty + slot), ((u / R) & 1) ^ 1, sm.abort_flag, p.err)) {
                    ok = false;
                    cc += c;  // uses issued so far in this tile
                    break;
                }
                ptx::mbar_arrive_expect_tx_elect(sm.bar(kBarFull + slot), bytes);
                ptx::tma_load_3d_elect(sm.slot(slot), kv_map, sm.bar(kBarFull + slot), c * 64, 0, phys0);
                if (live1)
                    ptx::tma_load_3d_elect(sm.slot(slot) + kPageChunkBytes, kv_map, sm.bar(kBarFull + slot), c * 64,
                                           0, phys1);
            }
            if (ok) cc += kChunks;
        }
    }
    if (!ok) {
        // Let every load this warp issued land before the CTA exits.
        const uint32_t first = cc > R ? cc - R : 0;
        for (uint32_t u = first; u < cc; ++u)
            warp_wait(sm.bar(kBarFull + static_cast<int>(u % R)), (u / R) & 1, sm.abort_flag, p.err, false);
    }
}

// -- tv score-MMA warp: S^T(t) into S buffer t & 1, chunk by chunk --------
template <int N, int SQ>
__device__ void tv_s_mma(const DecodeParams &p, const Range &w, const Smem &sm, uint32_t tmem)
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
            // the softmax has finished reading S^T(it - 2) from this buffer
            if (it >= 2 &&
                !(ok = warp_wait(sm.bar(kBarSEmpty + (it & 1)), ((it >> 1) & 1) ^ 1, sm.abort_flag, p.err)))
                break;
            ptx::tc_fence_after();
            const uint32_t d = tmem + C::S_COL + (it & 1) * N;
#pragma unroll 1
            for (int c = 0; c < kChunks; ++c) {
                const uint32_t u = cc + c;
                const int slot = static_cast<int>(u % R);
                if (!(ok = warp_wait(sm.bar(kBarFull + slot), (u / R) & 1, sm.abort_flag, p.err))) break;
                ptx::tc_fence_after();
                const uint32_t a0 = sm.slot(slot);
                const uint32_t b0 = sm.q + c * C::QCHUNK;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    ptx::mma_bf16_ss_elect(d, ptx::desc_sw128(a0 + 32u * k, 16, 1024),
                                           ptx::desc_sw128(b0 + 32u * k, 16, 1024), idS, (c | k) != 0);
                // a slot is free after three arrivals: this one and one
                // from each of the two transposer warps that read it; the
                // rope chunk is not transposed, so it takes all three here
                ptx::mma_commit_elect(sm.bar(kBarEmpty + slot));
                if (c == kChunks - 1) {
                    ptx::mma_commit_elect(sm.bar(kBarEmpty + slot));
                    ptx::mma_commit_elect(sm.bar(kBarEmpty + slot));
                }
            }
            if (!ok) break;
            ptx::mma_commit_elect(sm.bar(kBarSFull + (it & 1)));
            if (t == te - 1) ptx::mma_commit_elect(sm.bar(kBarQEmpty));
            cc += kChunks;
            ++it;
        }
    }
    ptx::mma_commit_elect(sm.bar(kBarDrain));
    warp_wait(sm.bar(kBarDrain), 0, sm.abort_flag, p.err, false);
}

// -- tv output-MMA warp: O^T += V^T (TMEM) . P^T (shared memory) ----------
template <int N, int SQ>
__device__ void tv_o_mma(const DecodeParams &p, const Range &w, const Smem &sm, uint32_t tmem)
{
    using C = Cfg<N, SQ>;
    constexpr uint32_t idO = ptx::idesc_bf16_f32(128, N, false, false);  // A in TMEM, P^T K-major
    uint32_t it = 0;
    bool ok = true;
    for (int b = w.b0; b <= w.b1 && ok; ++b) {
        const int L = max(0, __ldg(p.seqlens + b));
        const int nt = tiles_of(L);
        const int tb = (b == w.b0) ? w.t0 : 0;
        const int te = min((b == w.b1) ? w.t1 : nt, nt);
        for (int t = tb; t < te; ++t) {
            if (!(ok = warp_wait(sm.bar(kBarPFull), it & 1, sm.abort_flag, p.err))) break;
            if (!(ok = warp_wait(sm.bar(kBarVtFull), it & 1, sm.abort_flag, p.err))) break;
            ptx::tc_fence_after();
            const uint32_t pa = sm.p + (it & 1) * 2 * C::QCHUNK;
#pragma unroll 1
            for (int j = 0; j < 4; ++j) {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    ptx::mma_bf16_ts_elect(tmem + j * N, tmem + kVtCol + 64 * j + 8 * kk,
                                           ptx::desc_sw128(pa + (kk >> 2) * C::QCHUNK + 32u * (kk & 3), 16, 1024),
                                           idO, (t != tb) || (kk != 0));
            }
            ptx::mma_commit_elect(sm.bar(kBarODone));
            ++it;
        }
    }
    ptx::mma_commit_elect(sm.bar(kBarDrainO));
    warp_wait(sm.bar(kBarDrainO), 0, sm.abort_flag, p.err, false);
}

// -- tv transposer: 4 warps copy V(t) into TMEM as V^T --------------------
// Warp q owns TMEM lanes 32q..32q+31, i.e. latent dims 128j + 32q + (0..31)
// of every 128-dim block j: half of chunk 2j + q/2.  Per 16 dims x 16 tokens
// one ldmatrix.x4.trans feeds one tcgen05.st.16x256b.
template <int N, int SQ>
__device__ void tv_transposer(const DecodeParams &p, const Range &w, const Smem &sm, uint32_t tmem)
{
    const uint32_t R = static_cast<uint32_t>(p.ring);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = warp & 3;
    const int ttid = threadIdx.x - 192;  // 0..127 within the transposer group
    uint32_t cc = 0, it = 0, od = 0;
    bool ok = true;
    // ldmatrix row addresses: lane -> (matrix mi, row rr)
    const int mi = lane >> 3, rr = lane & 7;
    const int tok_in = rr + 8 * (mi & 1);        // token within a 16-token group
    const int dim_in = 8 * (mi >> 1);            // dim offset within a 16-dim half
    for (int b = w.b0; b <= w.b1 && ok; ++b) {
        const int L = max(0, __ldg(p.seqlens + b));
        const int nt = tiles_of(L);
        const int tb = (b == w.b0) ? w.t0 : 0;
        const int te = min((b == w.b1) ? w.t1 : nt, nt);
        for (int t = tb; t < te; ++t) {
            // V^T buffer free: the output MMA of the previous tile is complete
            bool good = true;
            while (od < it) {
                good = good && wait_bounded(sm.bar(kBarODone), od & 1, sm.abort_flag, p.err);
                ++od;
            }
            __syncwarp();
            if (!(ok = ptx::named_bar_and(2, 128, good))) break;
            ptx::tc_fence_after();
            const int valid = L - t * kTile;  // tokens of this tile inside the sequence
            // Warp q's share of chunk j (latent block j): 16 ldmatrix.x4 =
            // 64 registers.  All 16 loads of a chunk are in flight together,
            // and the next chunk's loads are issued before this chunk is
            // stored, so the shared-memory latency is paid about once per chunk.
            auto wait_chunk = [&](int j, uint32_t &slot_out) -> bool {
                const uint32_t u = cc + 2 * j + (q >> 1);
                slot_out = u % R;
                return warp_wait(sm.bar(kBarFull + static_cast<int>(slot_out)), (u / R) & 1, sm.abort_flag, p.err);
            };
            auto load_chunk = [&](uint32_t slot_id, uint32_t (&r)[64]) {
                const uint32_t sbase = sm.slot(static_cast<int>(slot_id));
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
            auto store_chunk = [&](int j, uint32_t (&r)[64]) {
                if (valid < kTile) {
                    // tokens past the sequence end: their P is zero, make V^T zero too
#pragma unroll
                    for (int h = 0; h < 2; ++h)
#pragma unroll
                        for (int gi = 0; gi < 8; ++gi)
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const int t0 = 16 * gi + 8 * (i & 1) + 2 * (lane & 3);
                                uint32_t &x = r[32 * h + 4 * gi + i];
                                if (t0 >= valid) x = 0;
                                else if (t0 + 1 >= valid) x &= 0xFFFFu;
                            }
                }
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int gg = 0; gg < 2; ++gg) {
                        uint32_t v[16];
#pragma unroll
                        for (int k = 0; k < 16; ++k) v[k] = r[32 * h + 16 * gg + k];
                        ptx::tmem_st_16x256b_x4(
                            tmem + (static_cast<uint32_t>(32 * q + 16 * h) << 16) + kVtCol + 64 * j + 32 * gg, v);
                    }
            };
            uint32_t ra[64], rb[64];
            uint32_t slot_a = 0, slot_b = 0;
            if (!(ok = wait_chunk(0, slot_a))) break;
            load_chunk(slot_a, ra);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t(&cur)[64] = (j & 1) ? rb : ra;
                uint32_t(&nxt)[64] = (j & 1) ? ra : rb;
                uint32_t &slot_cur = (j & 1) ? slot_b : slot_a;
                uint32_t &slot_nxt = (j & 1) ? slot_a : slot_b;
                if (j < 3) {
                    if (!(ok = wait_chunk(j + 1, slot_nxt))) break;
                    load_chunk(slot_nxt, nxt);
                }
                store_chunk(j, cur);
                // the stores consumed this chunk's loaded registers: release
                // this warp's share of the slot
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(sm.bar(kBarEmpty + static_cast<int>(slot_cur)));
            }
            if (!ok) break;
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            __syncwarp();
            ptx::named_bar_sync(2, 128);
            if (ttid == 0) ptx::mbar_arrive(sm.bar(kBarVtFull));
            cc += kChunks;
            ++it;
        }
    }
}

// -- tv softmax / epilogue: 4 warps, thread = one TMEM lane = one token row
template <int N, int SQ>
__device__ void tv_softmax(const DecodeParams &p, const Range &w, int g, const Smem &sm, uint32_t tmem)
{
    using C = Cfg<N, SQ>;
    constexpr int HG = C::HG;
    constexpr int NCH = C::NCH;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wq = warp & 3;              // TMEM lane quadrant this warp may access
    const int row = wq * 32 + lane;       // token row within the tile
    const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
    const int kp = tv_kpos(row);          // this row's K position in the output MMA
    const float NEG_INF = -INFINITY;
    uint32_t it = 0;   // tiles processed
    uint32_t od = 0;   // output-MMA completions observed
    bool ok = true;
    // Observe the output MMAs in order up to (not including) tile `upto`.
    auto observe_o = [&](uint32_t upto) -> bool {
        bool good = true;
        while (od < upto) {
            good = good && wait_bounded(sm.bar(kBarODone), od & 1, sm.abort_flag, p.err);
            ++od;
        }
        __syncwarp();
        return ptx::named_bar_and(1, 128, good);
    };

    for (int b = w.b0; b <= w.b1 && ok; ++b) {
        const int L = max(0, __ldg(p.seqlens + b));
        const int nt = tiles_of(L);
        const int tb = (b == w.b0) ? w.t0 : 0;
        const int te = min((b == w.b1) ? w.t1 : nt, nt);
        if (tb >= te) continue;
        const int split = (b == w.b0) ? w.split0 : 0;
        const int nvis0 = max(0, L - SQ + 1);  // tokens visible to query position 0
        float m[N], l[N];
#pragma unroll
        for (int n = 0; n < N; ++n) { m[n] = NEG_INF; l[n] = 0.f; }

        for (int t = tb; t < te; ++t) {
            const bool got_s = wait_bounded(sm.bar(kBarSFull + (it & 1)), (it >> 1) & 1, sm.abort_flag, p.err);
            __syncwarp();
            ok = ptx::named_bar_and(1, 128, got_s);
            if (!ok) break;
            ptx::tc_fence_after();
            const uint32_t s_taddr = tmem + lane_base + C::S_COL + (it & 1) * N;
            const int tok = t * kTile + row;
            const bool vis0 = tok < nvis0, vis1 = tok < L;
            float *red = sm.red + (it & 1) * 4 * N;
            // pass 1: masked log2-domain scores and their per-column maximum
            float sc[NCH][16];
#pragma unroll
            for (int ch = 0; ch < NCH; ++ch) {
                ptx::tmem_ld16(s_taddr + ch * 16, sc[ch]);
                ptx::tmem_wait_ld();
            }
            // S^T(it) is in registers: its TMEM buffer may be overwritten
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(sm.bar(kBarSEmpty + (it & 1)));
#pragma unroll
            for (int ch = 0; ch < NCH; ++ch) {
                float v[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int n = ch * 16 + e;
                    const bool vis = (SQ == 2 && n >= HG) ? vis1 : vis0;
                    sc[ch][e] = vis ? sc[ch][e] * p.scale_log2 : NEG_INF;
                    v[e] = sc[ch][e];
                }
                const float cmax = warp_colmax16(v, lane);
                if ((lane & 1) == 0) red[wq * N + ch * 16 + (lane >> 1)] = cmax;
            }
            __syncwarp();
            ptx::named_bar_sync(1, 128);
            // pass 2: running max, weights, P^T (permuted K order), running sums
            const uint32_t pa = sm.p + (it & 1) * 2 * C::QCHUNK + (kp >> 6) * C::QCHUNK;
            const uint32_t pcol = static_cast<uint32_t>(kp & 63);
            bool any_rescale = false;
            float alpha[N];
#pragma unroll
            for (int ch = 0; ch < NCH; ++ch) {
                float tmax[16];
                {
                    const float4 *r4 = reinterpret_cast<const float4 *>(red + ch * 16);
#pragma unroll
                    for (int e4 = 0; e4 < 4; ++e4) {
                        const float4 a0 = r4[e4], a1 = r4[N / 4 + e4], a2 = r4[2 * (N / 4) + e4],
                                     a3 = r4[3 * (N / 4) + e4];
                        tmax[4 * e4 + 0] = fmaxf(fmaxf(a0.x, a1.x), fmaxf(a2.x, a3.x));
                        tmax[4 * e4 + 1] = fmaxf(fmaxf(a0.y, a1.y), fmaxf(a2.y, a3.y));
                        tmax[4 * e4 + 2] = fmaxf(fmaxf(a0.z, a1.z), fmaxf(a2.z, a3.z));
                        tmax[4 * e4 + 3] = fmaxf(fmaxf(a0.w, a1.w), fmaxf(a2.w, a3.w));
                    }
                }
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int n = ch * 16 + e;
                    const float mnew = fmaxf(m[n], tmax[e]);
                    // The reference max follows the true running max, so the
                    // largest weight of a range is exactly 1.
                    const bool need = mnew > m[n];
                    alpha[n] = need ? ptx::ex2_approx(m[n] - mnew) : 1.f;
                    if (need) {
                        m[n] = mnew;
                        any_rescale = true;
                    }
                    const float mu = (m[n] == NEG_INF) ? 0.f : m[n];
                    const float pr = ptx::ex2_approx(sc[ch][e] - mu);  // masked entries: 2^-inf = 0
                    l[n] = l[n] * alpha[n] + pr;
                    const uint32_t addr = pa + n * 128u + ((((pcol >> 3) ^ static_cast<uint32_t>(n & 7)) << 4)) +
                                          ((pcol & 7u) << 1);
                    ptx::st_shared_b16(addr, __bfloat16_as_ushort(__float2bfloat16_rn(pr)));
                }
            }
            // The previous tile's output MMA must be complete before O^T is
            // rescaled (observed every tile, so the wait never lags).
            if (!(ok = observe_o(it))) break;
            ptx::tc_fence_after();
            if (any_rescale && t != tb) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
#pragma unroll
                    for (int ch = 0; ch < NCH; ++ch) {
                        float v[16];
                        const uint32_t ta = tmem + lane_base + j * N + ch * 16;
                        ptx::tmem_ld16(ta, v);
                        ptx::tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] *= alpha[ch * 16 + e];
                        ptx::tmem_st16(ta, v);
                    }
                }
                ptx::tmem_wait_st();
            }
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            ptx::mbar_arrive(sm.bar(kBarPFull));
            ++it;
        }
        if (!ok) break;
        if (!(ok = observe_o(it))) break;
        ptx::tc_fence_after();
        range_epilogue<N, SQ>(p, sm, tmem, b, split, g, m, l);
    }
}

// ============================================================== kernels
// Shared prologue of both variants: schedule check, shared-memory carve-up,
// barrier initialisation and TMEM allocation.  Returns false (uniformly) when
// this CTA has no work.
template <int N, int SQ>
__device__ __forceinline__ bool decode_setup(const DecodeParams &p, const CUtensorMap *kv_map,
                                             const CUtensorMap *q_map, uint8_t *smem_raw, Smem &sm, Range &w,
                                             uint32_t &tmem)
{
    using C = Cfg<N, SQ>;
    const int tuple = blockIdx.x / p.G;
    const int32_t *hdr = p.sched;
    if (hdr[1] != kSchedMagic || hdr[2] != p.B || hdr[3] != p.s_q || hdr[4] != p.H ||
        hdr[5] != p.num_sms || hdr[6] != p.num_tuples || hdr[7] != p.G) {
        if (threadIdx.x == 0) atomicOr(p.err, MLA_DEVERR_SCHEDULE);
        return false;
    }
    const int32_t *e = p.sched + kSchedHeader + tuple * kSchedEntry;
    w = Range{e[0], e[1], e[2], e[3], e[4]};
    if (w.b0 < 0 || w.b0 >= p.B || w.b1 < w.b0 || w.b1 >= p.B) return false;  // no work for this group

    const uint32_t raw = ptx::smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - raw);
    sm.ring = base;
    sm.q = base + p.ring * kSlotBytes;
    sm.p = sm.q + C::QBYTES;
    uint8_t *misc = gbase + p.ring * kSlotBytes + C::QBYTES + C::PBYTES;
    sm.bars = ptx::smem_addr(misc);
    sm.red = reinterpret_cast<float *>(misc + kMiscRedOffset);
    sm.lred = sm.red + 2 * 4 * N;
    sm.tmem_holder = reinterpret_cast<uint32_t *>(sm.lred + 4 * N);
    sm.abort_flag = reinterpret_cast<volatile int *>(sm.tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) {
        for (int s = 0; s < p.ring; ++s) {
            ptx::mbar_init(sm.bar(kBarFull + s), 1);
            ptx::mbar_init(sm.bar(kBarEmpty + s), C::TV ? 3 : 1);
        }
        ptx::mbar_init(sm.bar(kBarQFull), 1);
        ptx::mbar_init(sm.bar(kBarQEmpty), 1);
        ptx::mbar_init(sm.bar(kBarSFull), 1);
        ptx::mbar_init(sm.bar(kBarSFull + 1), 1);
        ptx::mbar_init(sm.bar(kBarSEmpty), 4);
        ptx::mbar_init(sm.bar(kBarSEmpty + 1), 4);
        ptx::mbar_init(sm.bar(kBarPFull), 128);
        ptx::mbar_init(sm.bar(kBarODone), 1);
        ptx::mbar_init(sm.bar(kBarVtFull), 1);
        ptx::mbar_init(sm.bar(kBarDrain), 1);
        ptx::mbar_init(sm.bar(kBarDrainO), 1);
        *sm.abort_flag = 0;
        ptx::fence_mbar_init();
        ptx::tma_prefetch_map(kv_map);
        ptx::tma_prefetch_map(q_map);
    }
    if (warp == 1) {
        ptx::tmem_alloc(ptx::smem_addr(sm.tmem_holder), C::TMEM_COLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    tmem = *sm.tmem_holder;
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

template <int N, int SQ>
__global__ void __launch_bounds__(kThreadsSS, 1)
mla_decode_ss_kernel(const __grid_constant__ CUtensorMap kv_map, const __grid_constant__ CUtensorMap q_map,
                     const DecodeParams p)
{
    extern __shared__ uint8_t smem_raw[];
    Smem sm;
    Range w;
    uint32_t tmem;
    ptx::griddep_launch_dependents();
    if (!decode_setup<N, SQ>(p, &kv_map, &q_map, smem_raw, sm, w, tmem)) return;
    const int warp = threadIdx.x >> 5;
    const int g = blockIdx.x % p.G;
    if (warp == 0) ss_producer<N, SQ>(p, w, g, sm, &kv_map, &q_map);
    else if (warp == 1) ss_mma<N, SQ>(p, w, sm, tmem);
    else ss_softmax<N, SQ>(p, w, g, sm, tmem);
    decode_teardown<N, SQ>(tmem);
}

template <int N, int SQ>
__global__ void __launch_bounds__(kThreadsTV, 1)
mla_decode_tv_kernel(const __grid_constant__ CUtensorMap kv_map, const __grid_constant__ CUtensorMap q_map,
                     const DecodeParams p)
{
    extern __shared__ uint8_t smem_raw[];
    Smem sm;
    Range w;
    uint32_t tmem;
    ptx::griddep_launch_dependents();
    if (!decode_setup<N, SQ>(p, &kv_map, &q_map, smem_raw, sm, w, tmem)) return;
    const int warp = threadIdx.x >> 5;
    const int g = blockIdx.x % p.G;
    if (warp == 0) tv_producer<N, SQ>(p, w, g, sm, &kv_map, &q_map);
    else if (warp == 1) tv_s_mma<N, SQ>(p, w, sm, tmem);
    else if (warp < 6) tv_softmax<N, SQ>(p, w, g, sm, tmem);
    else if (warp < 10) tv_transposer<N, SQ>(p, w, sm, tmem);
    else tv_o_mma<N, SQ>(p, w, sm, tmem);
    decode_teardown<N, SQ>(tmem);
}

// =============================================================== combine
// One 128-thread block per output row (b, i, h) of a sequence cut into pieces.
// The pieces' lse values go to shared memory once; each thread then owns four
// latent dims and issues its loads of every piece unrolled, so the partials
// (fresh in L2) are fetched with all loads in flight instead of one piece at a
// time.  Launched as a programmatic dependent of the attention kernel: it may
// become resident early and waits in hardware for that grid to finish.
constexpr int kCombineThreads = 128;

__global__ void __launch_bounds__(kCombineThreads)
mla_combine_kernel(const int32_t *__restrict__ split_base, const float *__restrict__ ws_o,
                   const float *__restrict__ ws_lse, int B, int s_q, int H, int HG, int G, int max_pieces,
                   uint16_t *__restrict__ out, float *__restrict__ lse, int32_t *__restrict__ err)
{
    constexpr int kBatch = 16;  // pieces whose loads are in flight together
    ptx::griddep_wait();        // the attention grid (and its memory) is complete
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
    const float *lsrc = ws_lse + row0;
    const float4 *src = reinterpret_cast<const float4 *>(ws_o + row0 * kDV) + tid;
    const int64_t step = pstride * kDV / 4;  // float4s between consecutive pieces
    // Every thread reads all piece lse values itself (broadcast loads) together
    // with its own partials, so the merge costs one round trip per batch.
    float M = -INFINITY;
    for (int k = 0; k < n; ++k) M = fmaxf(M, lsrc[k * pstride]);
    if (M == -INFINITY) {  // every piece saw no token
        *o = make_uint2(0, 0);
        if (tid == 0) lse[r] = -INFINITY;
        return;
    }
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float ssum = 0.f;
    for (int k0 = 0; k0 < n; k0 += kBatch) {
        float4 x[kBatch];
        float lk[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            if (k0 + u < n) {
                x[u] = src[(k0 + u) * step];
                lk[u] = lsrc[(k0 + u) * pstride];
            }
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            if (k0 + u < n) {
                const float wk = expf(lk[u] - M);
                ssum += wk;
                acc.x += wk * x[u].x;
                acc.y += wk * x[u].y;
                acc.z += wk * x[u].z;
                acc.w += wk * x[u].w;
            }
        }
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

bool resolve(int s_q, int H, Shape *s)
{
    if (s_q != 1 && s_q != 2) return false;
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

struct DeviceInfo {
    int smem_optin = 0;
    int major = 0;
    bool attr_set[8] = {false, false, false, false, false, false, false, false};
};

std::mutex g_dev_mutex;
DeviceInfo g_dev[64];

template <int N, int SQ>
int kernel_index()
{
    if (N == 16 && SQ == 1) return 0;
    if (N == 32 && SQ == 1) return 1;
    if (N == 32 && SQ == 2) return 2;
    if (N == 64 && SQ == 1) return 3;
    return 4;
}

template <int N, int SQ>
int ring_for(int smem_optin, size_t *smem_bytes)
{
    using C = Cfg<N, SQ>;
    const int fixed = static_cast<int>(C::QBYTES + C::PBYTES + misc_bytes<N>() + 1024);
    int R = (smem_optin - fixed) / static_cast<int>(kSlotBytes);
    if (R > kMaxRing) R = kMaxRing;
    *smem_bytes = static_cast<size_t>(fixed) + static_cast<size_t>(R) * kSlotBytes;
    return R;
}

template <int N, int SQ>
mla_status_t launch_decode(const CUtensorMap &kv_map, const CUtensorMap &q_map, DecodeParams prm, int grid,
                           cudaStream_t stream)
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
    const int R = ring_for<N, SQ>(info.smem_optin, &smem);
    if (R < kMinRing) {
        snprintf(g_last_error, sizeof g_last_error, "not enough shared memory for a %d-slot ring", kMinRing);
        return MLA_ERR_CUDA;
    }
    const int ki = kernel_index<N, SQ>();
    void (*kernel)(const CUtensorMap, const CUtensorMap, const DecodeParams);
    if constexpr (Cfg<N, SQ>::TV)
        kernel = mla_decode_tv_kernel<N, SQ>;
    else
        kernel = mla_decode_ss_kernel<N, SQ>;
    if (!info.attr_set[ki]) {
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
        std::lock_guard<std::mutex> lock(g_dev_mutex);
        g_dev[dev].attr_set[ki] = true;
    }
    prm.ring = R;
    kernel<<<grid, Cfg<N, SQ>::THREADS, smem, stream>>>(kv_map, q_map, prm);
    e = cudaGetLastError();
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

}  // namespace host
}  // namespace mla

using namespace mla;
using namespace mla::host;

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
    if (!cache_seqlens || !sched_meta || !num_splits) return MLA_ERR_INVALID_ARG;
    if (B < 1 || B > kMaxBatch) return MLA_ERR_INVALID_ARG;
    Shape sh;
    if (!resolve(s_q, H, &sh)) return MLA_ERR_UNSUPPORTED_SHAPE;
    if (num_sms < sh.G || num_sms > kMaxSms) return MLA_ERR_UNSUPPORTED_SHAPE;
    if ((reinterpret_cast<uintptr_t>(cache_seqlens) | reinterpret_cast<uintptr_t>(sched_meta) |
         reinterpret_cast<uintptr_t>(num_splits)) & 3)
        return MLA_ERR_MISALIGNED;
    const int tuples = num_sms / sh.G;
    mla_metadata_kernel<<<1, kMetaThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        cache_seqlens, B, s_q, H, num_sms, tuples, sh.G, sched_meta, num_splits);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "mla_metadata_kernel launch");
    return MLA_OK;
}

mla_status_t mla_decode_combine(const int32_t *num_splits, const int32_t *sched_meta, const void *workspace,
                                size_t workspace_bytes, int B, int s_q, int H, int num_sms, uint16_t *out,
                                float *lse, void *stream)
{
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
    cudaError_t e = cudaLaunchKernelEx(&cfg, mla_combine_kernel, num_splits, ws_o, ws_lse, B, s_q, H, sh.HG, sh.G,
                                       wl.pieces, out, lse, const_cast<int32_t *>(sched_meta));
    if (e != cudaSuccess) return cuda_fail(e, "mla_combine_kernel launch");
    return MLA_OK;
}

mla_status_t mla_decode_attention(const uint16_t *q, const uint16_t *kv_cache, const int32_t *block_table,
                        const int32_t *cache_seqlens, int B, int s_q, int H, int64_t num_blocks, int max_blocks,
                        float softmax_scale, int num_sms, const int32_t *sched_meta, const int32_t *num_splits,
                        void *workspace, size_t workspace_bytes, uint16_t *out, float *lse, void *stream)
{
    if (!q || !kv_cache || !block_table || !cache_seqlens || !sched_meta || !num_splits || !workspace || !out ||
        !lse)
        return MLA_ERR_INVALID_ARG;
    if (B < 1 || B > kMaxBatch || num_blocks < 1 || num_blocks > INT32_MAX || max_blocks < 1)
        return MLA_ERR_INVALID_ARG;
    if (!std::isfinite(softmax_scale)) return MLA_ERR_INVALID_ARG;
    Shape sh;
    if (!resolve(s_q, H, &sh)) return MLA_ERR_UNSUPPORTED_SHAPE;
    if (num_sms < sh.G || num_sms > kMaxSms) return MLA_ERR_UNSUPPORTED_SHAPE;
    if ((reinterpret_cast<uintptr_t>(q) & 15) || (reinterpret_cast<uintptr_t>(kv_cache) & 15) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255) || (reinterpret_cast<uintptr_t>(out) & 7) ||
        (reinterpret_cast<uintptr_t>(lse) & 3) || (reinterpret_cast<uintptr_t>(block_table) & 3) ||
        (reinterpret_cast<uintptr_t>(cache_seqlens) & 3) || (reinterpret_cast<uintptr_t>(sched_meta) & 3) ||
        (reinterpret_cast<uintptr_t>(num_splits) & 3))
        return MLA_ERR_MISALIGNED;
    const WorkspaceLayout wl = layout(B, s_q, sh, num_sms);
    if (workspace_bytes < wl.total) return MLA_ERR_WORKSPACE_TOO_SMALL;
    if (static_cast<int64_t>(B) * s_q * H > INT32_MAX) return MLA_ERR_INVALID_ARG;

    EncodeTiledFn encode = encode_fn();
    if (!encode) {
        snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled unavailable");
        return MLA_ERR_CUDA;
    }
    // kv_cache viewed as [num_blocks][64 rows][576 cols]; box 64 cols x 64 rows x 1 block.
    CUtensorMap kv_map, q_map;
    {
        const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kDQK), static_cast<cuuint64_t>(kPage),
                                    static_cast<cuuint64_t>(num_blocks)};
        const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kDQK) * 2, static_cast<cuuint64_t>(kPage) * kDQK * 2};
        const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(kPage), 1};
        const cuuint32_t estr[3] = {1, 1, 1};
        const CUresult r = encode(&kv_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t *>(kv_cache), dims,
                                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) {
            snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled(kv) failed: %d", static_cast<int>(r));
            return MLA_ERR_CUDA;
        }
    }
    // q viewed as [B * s_q * H rows][576 cols]; box 64 cols x (heads per CTA) rows.
    {
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kDQK), static_cast<cuuint64_t>(B) * s_q * H};
        const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kDQK) * 2};
        const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(sh.HG)};
        const cuuint32_t estr[2] = {1, 1};
        const CUresult r = encode(&q_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t *>(q), dims,
                                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) {
            snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled(q) failed: %d", static_cast<int>(r));
            return MLA_ERR_CUDA;
        }
    }

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
    const int grid = prm.num_tuples * sh.G;
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    mla_status_t rc;
    if (sh.N == 16) rc = launch_decode<16, 1>(kv_map, q_map, prm, grid, st);
    else if (sh.N == 32 && s_q == 1) rc = launch_decode<32, 1>(kv_map, q_map, prm, grid, st);
    else if (sh.N == 32) rc = launch_decode<32, 2>(kv_map, q_map, prm, grid, st);
    else if (s_q == 1) rc = launch_decode<64, 1>(kv_map, q_map, prm, grid, st);
    else rc = launch_decode<64, 2>(kv_map, q_map, prm, grid, st);
    return rc;
}

mla_status_t mla_decode(const uint16_t *q, const uint16_t *kv_cache, const int32_t *block_table,
                        const int32_t *cache_seqlens, int B, int s_q, int H, int64_t num_blocks, int max_blocks,
                        float softmax_scale, int num_sms, const int32_t *sched_meta, const int32_t *num_splits,
                        void *workspace, size_t workspace_bytes, uint16_t *out, float *lse, void *stream)
{
    const mla_status_t rc =
        mla_decode_attention(q, kv_cache, block_table, cache_seqlens, B, s_q, H, num_blocks, max_blocks,
                             softmax_scale, num_sms, sched_meta, num_splits, workspace, workspace_bytes, out, lse,
                             stream);
    if (rc != MLA_OK) return rc;
    return mla_decode_combine(num_splits, sched_meta, workspace, workspace_bytes, B, s_q, H, num_sms, out, lse,
                              stream);
}

mla_status_t mla_decode_static_workspace(const uint16_t *q, const uint16_t *kv_cache, const int32_t *block_table,
                                         const int32_t *cache_seqlens, int B, int s_q, int H, int64_t num_blocks,
                                         int max_blocks, float softmax_scale, int num_sms,
                                         const int32_t *sched_meta, const int32_t *num_splits, uint16_t *out,
                                         float *lse, void *stream)
{
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

mla_status_t mla_get_device_error(const int32_t *sched_meta, int32_t *host_code, void *stream)
{
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
