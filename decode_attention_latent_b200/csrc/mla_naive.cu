// mla_naive.cu -- MLA decode in non-absorbed form for B200 (sm_100a).
//
// The latent cache is the one the absorbed kernel reads (per token 512 latent
// columns C, then 64 rope columns), but each head keeps its own 128-wide keys
// and values, decompressed from C tile by tile as "FlashMLA: compressing the
// KV cache to one eighth" (jsqmd.com) describes in "FlashMLA compute flow",
// steps 1-5:
//     K_tile = C_tile W_UK,   V_tile = C_tile W_UV        (per head)
//     S = Q K^T,   online softmax,   O += softmax(S) V.
// Per head h and token j:  k_j = [C_j W_UK[h]^T (128), rope_j (64)],
// v_j = C_j W_UV[h]^T (128), with the matrices stored [H][128][512] (row e of
// head h holds the latent coefficients of dimension e).
//
// One CTA per (sequence, head, split of the sequence's tiles).  Per 128-token
// tile the two up-projections run on the tensor cores, both with K-major
// operands straight from TMA-swizzled shared memory:
//     K^T-side:  D_K [128 tokens x 128 e]  = C [tokens x 512] . W_UK[h]^T
//     V-side:    D_V^T [128 e x 128 tokens] = W_UV[h] [e x 512] . C^T
// (M = 128, N = 128, K = 512 in 64-column chunks), accumulating in fp32 in
// TMEM (two buffers, so the next tile's products overlap this tile's
// softmax).  The rest is small and stays in fp32 on the CUDA cores: thread r
// of the four math warps owns TMEM lane r, so it reads token r's key row for
// the scores and value dimension r's row of V^T (all 128 tokens) for the
// output, with the tile's weights broadcast from shared memory.  No
// decompressed key or value is rounded below fp32.  Splits of a sequence are
// merged through their log-sum-exps by mla_naive_combine_kernel.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/mla_decode.h"
#include "sm100_ptx.cuh"

namespace mla {
namespace host {
extern thread_local char g_last_error[256];
mla_status_t cuda_fail(cudaError_t e, const char *what);
bool tensor_map(CUtensorMap *out, const char *what, CUtensorMapDataType dtype, int rank, const void *ptr,
                const cuuint64_t *dims, const cuuint64_t *strides, const cuuint32_t *box, CUtensorMapSwizzle swizzle,
                CUtensorMapL2promotion promo);
void clear_error();
}  // namespace host

namespace naive {

constexpr int kTile = MLA_TILE;                 // tokens per tile (two pages)
constexpr int kPage = MLA_PAGE;
constexpr int kLat = MLA_D_V;                   // latent columns
constexpr int kE = MLA_NAIVE_D;                 // decompressed key / value width
constexpr int kRope = MLA_D_QK - MLA_D_V;       // 64 rope columns
constexpr int kDq = kE + kRope;                 // 192-wide queries
constexpr int kLatChunks = kLat / 64;           // 8 chunks of 64 latent columns
constexpr uint32_t kChunk = 16384;              // 128 rows x 64 bf16, 128-byte swizzled
constexpr uint32_t kPageChunk = 8192;
constexpr uint32_t kStage = 3 * kChunk;         // C chunk | W_UK chunk | W_UV chunk
constexpr int kStages = 3;
constexpr int kThreads = 192;                   // producer, MMA, 4 math warps
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr int kMaxSplits = 4096;

// barriers
constexpr int kBarFull = 0;                     // [kStages]
constexpr int kBarEmpty = kStages;              // [kStages]
constexpr int kBarRFull = 2 * kStages;          // [2] rope chunk of a tile loaded
constexpr int kBarREmpty = kBarRFull + 2;       // [2] rope chunk read (4 math warps)
constexpr int kBarTFull = kBarREmpty + 2;       // [2] D_K and D_V^T of a tile complete
constexpr int kBarTEmpty = kBarTFull + 2;       // [2] TMEM buffer read (4 math warps)
constexpr int kBarDrain = kBarTEmpty + 2;
constexpr int kNumBars = kBarDrain + 1;

struct Params {
    const int32_t *block_table;
    const int32_t *seqlens;
    const uint16_t *q;  // [B, s_q, H, 192]
    float *ws_o;        // [pieces][s_q][128]
    float *ws_lse;      // [pieces][s_q]
    int32_t *err;
    int B, H, splits, tiles_per_split, max_blocks;
    int64_t num_blocks;
    float scale;
};

// Bounded mbarrier wait: gives up after kWaitLimitNs (setting the abort flag
// and MLA_DEVERR_TIMEOUT), or at once when another role has aborted unless
// `honour_abort` is false (a drain that must see its own work complete).
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int *abort_flag, int32_t *err,
                                             bool honour_abort = true)
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

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag, int32_t *err)
{
    return __all_sync(0xffffffffu, wait_bounded(bar, parity, abort_flag, err));
}

// Physical block of page `page` of sequence b (0, with an error bit, for an
// entry outside the cache).
__device__ __forceinline__ int page_block(const Params &p, int b, int page)
{
    if (page >= p.max_blocks) {
        atomicOr(p.err, MLA_DEVERR_SEQLEN);
        return 0;
    }
    const int id = __ldg(p.block_table + static_cast<int64_t>(b) * p.max_blocks + page);
    if (id < 0 || static_cast<int64_t>(id) >= p.num_blocks) {
        atomicOr(p.err, MLA_DEVERR_BLOCK_TABLE);
        return 0;
    }
    return id;
}

template <int SQ>
__global__ void __launch_bounds__(kThreads, 1)
mla_naive_kernel(const __grid_constant__ CUtensorMap kv_map, const __grid_constant__ CUtensorMap wk_map,
                 const __grid_constant__ CUtensorMap wv_map, const Params p)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = ptx::smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - raw);
    const uint32_t stages = base;                         // kStages x 48 KB
    const uint32_t rope = base + kStages * kStage;        // 2 x 16 KB
    float *qs = reinterpret_cast<float *>(gbase + kStages * kStage + 2 * kChunk);  // [SQ][192]
    float *ps = qs + SQ * kDq;                            // [SQ][128] weights of a tile
    float *red = ps + SQ * kTile;                         // [2][4][SQ] warp maxima, [2][4][SQ] warp sums
    uint64_t *bars = reinterpret_cast<uint64_t *>(red + 16 * SQ + 16);
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(bars + kNumBars);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);
    const uint32_t bar0 = ptx::smem_addr(bars);
    auto bar = [&](int i) { return bar0 + 8u * i; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int split = blockIdx.x % p.splits;
    const int h = (blockIdx.x / p.splits) % p.H;
    const int b = blockIdx.x / (p.splits * p.H);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(bar(kBarFull + s), 1);
            ptx::mbar_init(bar(kBarEmpty + s), 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(bar(kBarRFull + i), 1);
            ptx::mbar_init(bar(kBarREmpty + i), 4);
            ptx::mbar_init(bar(kBarTFull + i), 1);
            ptx::mbar_init(bar(kBarTEmpty + i), 4);
        }
        ptx::mbar_init(bar(kBarDrain), 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
        ptx::tma_prefetch_map(&kv_map);
        ptx::tma_prefetch_map(&wk_map);
        ptx::tma_prefetch_map(&wv_map);
    }
    if (warp == 1) {
        ptx::tmem_alloc(ptx::smem_addr(tmem_holder), 512);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    int L = __ldg(p.seqlens + b);
    if (L < 0) {
        if (threadIdx.x == 0) atomicOr(p.err, MLA_DEVERR_SEQLEN);
        L = 0;
    }
    const int nt = (L + kTile - 1) / kTile;
    const int t0 = split * p.tiles_per_split;
    const int t1 = min(nt, t0 + p.tiles_per_split);
    const int ntile = max(0, t1 - t0);

    if (warp == 0) {
        // ---- producer: per tile the rope chunk, then 8 stages of
        // (C chunk, W_UK chunk, W_UV chunk); a stage's C chunk holds the
        // tile's two pages (rows 0-63 and 64-127).
        uint32_t su = 0;
        int rope_uses = 0;
        bool ok = true;
        for (int u = 0; u < ntile && ok; ++u) {
            const int t = t0 + u;
            const int phys0 = page_block(p, b, 2 * t);
            const bool live1 = t * kTile + kPage < L;
            const int phys1 = live1 ? page_block(p, b, 2 * t + 1) : 0;
            const uint32_t cb = live1 ? 2 * kPageChunk : kPageChunk;
            const int rb = u & 1;
            if (!(ok = warp_wait(bar(kBarREmpty + rb), ((u >> 1) & 1) ^ 1, abort_flag, p.err))) break;
            ptx::mbar_arrive_expect_tx_elect(bar(kBarRFull + rb), cb);
            ptx::tma_load_3d_elect(rope + rb * kChunk, &kv_map, bar(kBarRFull + rb), kLat, 0, phys0);
            if (live1) ptx::tma_load_3d_elect(rope + rb * kChunk + kPageChunk, &kv_map, bar(kBarRFull + rb), kLat, 0, phys1);
            ++rope_uses;
            for (int c = 0; c < kLatChunks; ++c, ++su) {
                const int s = static_cast<int>(su % kStages);
                if (!(ok = warp_wait(bar(kBarEmpty + s), ((su / kStages) & 1) ^ 1, abort_flag, p.err))) break;
                const uint32_t dst = stages + s * kStage;
                ptx::mbar_arrive_expect_tx_elect(bar(kBarFull + s), cb + 2 * kChunk);
                ptx::tma_load_3d_elect(dst, &kv_map, bar(kBarFull + s), 64 * c, 0, phys0);
                if (live1) ptx::tma_load_3d_elect(dst + kPageChunk, &kv_map, bar(kBarFull + s), 64 * c, 0, phys1);
                ptx::tma_load_2d_elect(dst + kChunk, &wk_map, bar(kBarFull + s), 64 * c, h * kE);
                ptx::tma_load_2d_elect(dst + 2 * kChunk, &wv_map, bar(kBarFull + s), 64 * c, h * kE);
            }
        }
        if (!ok) {
            // let the loads issued land before the CTA exits: the last
            // kStages stage uses and the last two rope chunks
            const uint32_t first = su > kStages ? su - kStages : 0;
            for (uint32_t x = first; x < su; ++x)
                wait_bounded(bar(kBarFull + static_cast<int>(x % kStages)), (x / kStages) & 1, abort_flag, p.err,
                             false);
            for (int x = max(0, rope_uses - 2); x < rope_uses; ++x)
                wait_bounded(bar(kBarRFull + (x & 1)), (x >> 1) & 1, abort_flag, p.err, false);
        }
    } else if (warp == 1) {
        // ---- MMA issue: D_K = C . W_UK^T and D_V^T = W_UV . C^T per tile,
        // into TMEM buffer u % 2 (D_K in its first 128 columns, D_V^T next)
        constexpr uint32_t idesc = ptx::idesc_bf16_f32(128, 128, false, false);
        uint32_t su = 0;
        bool ok = true;
        for (int u = 0; u < ntile && ok; ++u) {
            const int tb = u & 1;
            if (u >= 2 && !(ok = warp_wait(bar(kBarTEmpty + tb), ((u >> 1) & 1) ^ 1, abort_flag, p.err))) break;
            ptx::tc_fence_after();
            const uint32_t dk = tmem + 256u * tb, dv = dk + 128u;
            for (int c = 0; c < kLatChunks; ++c, ++su) {
                const int s = static_cast<int>(su % kStages);
                if (!(ok = warp_wait(bar(kBarFull + s), (su / kStages) & 1, abort_flag, p.err))) break;
                ptx::tc_fence_after();
                const uint32_t ca = stages + s * kStage, wka = ca + kChunk, wva = ca + 2 * kChunk;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t acc = (c | k) != 0;
                    ptx::mma_bf16_ss_elect(dk, ptx::desc_sw128(ca + 32u * k, 16, 1024),
                                           ptx::desc_sw128(wka + 32u * k, 16, 1024), idesc, acc);
                    ptx::mma_bf16_ss_elect(dv, ptx::desc_sw128(wva + 32u * k, 16, 1024),
                                           ptx::desc_sw128(ca + 32u * k, 16, 1024), idesc, acc);
                }
                ptx::mma_commit_elect(bar(kBarEmpty + s));
            }
            if (!ok) break;
            ptx::mma_commit_elect(bar(kBarTFull + tb));
        }
        ptx::mma_commit_elect(bar(kBarDrain));
        wait_bounded(bar(kBarDrain), 0, abort_flag, p.err, false);  // every issued MMA complete before dealloc
    } else {
        // ---- math warps: thread r owns TMEM lane r (warp quadrant rules:
        // warp w reads lanes 32 (w % 4) .. +31)
        const int r = 32 * (warp & 3) + lane;
        const int tid = threadIdx.x - 64;
        const uint32_t lane_base = static_cast<uint32_t>(32 * (warp & 3)) << 16;
        const uint16_t *qg = p.q + ((static_cast<int64_t>(b) * SQ) * p.H + h) * kDq;
        for (int x = tid; x < SQ * kDq; x += 128) {
            const int i = x / kDq, d = x % kDq;
            qs[x] = __bfloat162float(__ushort_as_bfloat16(qg[static_cast<int64_t>(i) * p.H * kDq + d]));
        }
        ptx::named_bar_sync(1, 128);
        float m[SQ], l[SQ], o[SQ];
#pragma unroll
        for (int i = 0; i < SQ; ++i) {
            m[i] = -INFINITY;
            l[i] = 0.f;
            o[i] = 0.f;
        }
        bool ok = true;
        for (int u = 0; u < ntile; ++u) {
            const int t = t0 + u;
            const int tok = t * kTile + r;
            const int valid = min(kTile, L - t * kTile);  // tokens of this tile inside the sequence
            // rope part of token r's score: row r of the rope chunk (128-byte
            // swizzled: 16-byte unit x of row r sits at unit x ^ (r % 8))
            const int rb = u & 1;
            ok = warp_wait(bar(kBarRFull + rb), (u >> 1) & 1, abort_flag, p.err) && ok;
            float sc[SQ];
#pragma unroll
            for (int i = 0; i < SQ; ++i) sc[i] = 0.f;
            {
                const uint32_t row = rope + rb * kChunk + static_cast<uint32_t>(r) * 128u;
#pragma unroll
                for (int x = 0; x < 8; ++x) {
                    const uint4 w4 = ptx::ld_shared_v4(row + ((static_cast<uint32_t>(x) ^ (r & 7)) << 4));
                    const uint32_t wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const float lo = __uint_as_float(wv[k] << 16), hi = __uint_as_float(wv[k] & 0xFFFF0000u);
#pragma unroll
                        for (int i = 0; i < SQ; ++i)
                            sc[i] = fmaf(lo, qs[i * kDq + kE + 8 * x + 2 * k],
                                         fmaf(hi, qs[i * kDq + kE + 8 * x + 2 * k + 1], sc[i]));
                    }
                }
            }
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar(kBarREmpty + rb));
            // key part: token r's row of D_K
            const int tb = u & 1;
            ok = warp_wait(bar(kBarTFull + tb), (u >> 1) & 1, abort_flag, p.err) && ok;
            ptx::tc_fence_after();
            const uint32_t dk = tmem + lane_base + 256u * tb, dv = dk + 128u;
#pragma unroll 1
            for (int c0 = 0; c0 < kE; c0 += 32) {
                float kv[32];
                ptx::tmem_ld32(dk + c0, kv);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e)
#pragma unroll
                    for (int i = 0; i < SQ; ++i) sc[i] = fmaf(kv[e], qs[i * kDq + c0 + e], sc[i]);
            }
            // scores, masked: query i sees tokens < L - SQ + 1 + i
            float s[SQ], pw[SQ];
#pragma unroll
            for (int i = 0; i < SQ; ++i) {
                const bool vis = tok < L - SQ + 1 + i;
                s[i] = vis ? sc[i] * p.scale : -INFINITY;
            }
            // tile maximum and running maximum per query column
            float *rm = red + (u & 1) * 8 * SQ;
#pragma unroll
            for (int i = 0; i < SQ; ++i) {
                float x = s[i];
#pragma unroll
                for (int k = 16; k > 0; k >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, k));
                if (lane == 0) rm[(warp & 3) * SQ + i] = x;
            }
            ptx::named_bar_sync(1, 128);
            float alpha[SQ];
#pragma unroll
            for (int i = 0; i < SQ; ++i) {
                const float tm = fmaxf(fmaxf(rm[i], rm[SQ + i]), fmaxf(rm[2 * SQ + i], rm[3 * SQ + i]));
                const float mn = fmaxf(m[i], tm);
                alpha[i] = (m[i] == -INFINITY) ? 0.f : expf(m[i] - mn);
                pw[i] = (s[i] == -INFINITY) ? 0.f : expf(s[i] - mn);
                m[i] = mn;
                float x = pw[i];
#pragma unroll
                for (int k = 16; k > 0; k >>= 1) x += __shfl_xor_sync(0xffffffffu, x, k);
                if (lane == 0) rm[4 * SQ + (warp & 3) * SQ + i] = x;
                ps[i * kTile + r] = pw[i];
            }
            ptx::named_bar_sync(1, 128);
#pragma unroll
            for (int i = 0; i < SQ; ++i)
                l[i] = alpha[i] * l[i] + ((rm[4 * SQ + i] + rm[5 * SQ + i]) + (rm[6 * SQ + i] + rm[7 * SQ + i]));
            // output: value dimension r over the tile's tokens (row r of D_V^T);
            // tokens past the sequence end are skipped, whatever they hold
            float acc[SQ];
#pragma unroll
            for (int i = 0; i < SQ; ++i) acc[i] = 0.f;
#pragma unroll 1
            for (int c0 = 0; c0 < kTile; c0 += 32) {
                float vv[32];
                ptx::tmem_ld32(dv + c0, vv);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const bool in = c0 + e < valid;
#pragma unroll
                    for (int i = 0; i < SQ; ++i) {
                        const float prod = ps[i * kTile + c0 + e] * vv[e];
                        acc[i] += in ? prod : 0.f;
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < SQ; ++i) o[i] = alpha[i] * o[i] + acc[i];
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar(kBarTEmpty + tb));
            // the four math warps leave together (their named barriers need all 128 threads)
            if (!ptx::named_bar_and(1, 128, ok)) break;
        }
        // this split's piece: O / l (fp32) and lse, or an empty state
        const int64_t piece = blockIdx.x;
#pragma unroll
        for (int i = 0; i < SQ; ++i) {
            const bool any = l[i] > 0.f;
            p.ws_o[(piece * SQ + i) * kE + r] = any ? o[i] / l[i] : 0.f;
            if (r == 0) p.ws_lse[piece * SQ + i] = any ? m[i] + logf(l[i]) : -INFINITY;
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 512);
    }
}

// One warp per output row (b, i, h): the row's splits merged through their
// log-sum-exps, each lane owning four of the 128 value dimensions.
__global__ void __launch_bounds__(128)
mla_naive_combine_kernel(const float *__restrict__ ws_o, const float *__restrict__ ws_lse, int B, int s_q, int H,
                         int splits, uint16_t *__restrict__ out, float *__restrict__ lse)
{
    const int lane = threadIdx.x & 31;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * 4 + (threadIdx.x >> 5);
    if (row >= static_cast<int64_t>(B) * s_q * H) return;
    const int h = static_cast<int>(row % H);
    const int i = static_cast<int>((row / H) % s_q);
    const int64_t b = row / (static_cast<int64_t>(H) * s_q);
    const int64_t p0 = (b * H + h) * splits;  // first piece of (b, h)
    float M = -INFINITY;
    for (int s = lane; s < splits; s += 32) M = fmaxf(M, ws_lse[(p0 + s) * s_q + i]);
#pragma unroll
    for (int k = 16; k > 0; k >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, k));
    uint2 *dst = reinterpret_cast<uint2 *>(out + row * kE) + lane;
    if (M == -INFINITY) {
        *dst = make_uint2(0, 0);
        if (lane == 0) lse[row] = -INFINITY;
        return;
    }
    float z = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < splits; ++s) {
        const float ls = ws_lse[(p0 + s) * s_q + i];
        if (ls == -INFINITY) continue;  // uniform across the warp
        const float w = expf(ls - M);
        const float4 v = reinterpret_cast<const float4 *>(ws_o + ((p0 + s) * s_q + i) * kE)[lane];
        z += w;
        acc.x = fmaf(w, v.x, acc.x);
        acc.y = fmaf(w, v.y, acc.y);
        acc.z = fmaf(w, v.z, acc.z);
        acc.w = fmaf(w, v.w, acc.w);
    }
    const float inv = 1.f / z;
    __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
    __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
    uint2 packed;
    memcpy(&packed.x, &lo, 4);
    memcpy(&packed.y, &hi, 4);
    *dst = packed;
    if (lane == 0) lse[row] = M + logf(z);
}

// ------------------------------------------------------------------- host
struct Split {
    int splits, tiles_per_split;
};

// Splits per sequence: the longest possible sequence (max_blocks pages) cut
// so that B x H x splits CTAs make about eight waves over num_sms SMs.
Split split_for(int B, int H, int max_blocks, int num_sms)
{
    const int64_t max_tiles = (static_cast<int64_t>(max_blocks) + 1) / 2;
    const int64_t units = max_tiles * B * H;
    const int64_t target = 8ll * num_sms;
    int64_t tps = (units + target - 1) / target;
    if (tps < 1) tps = 1;
    if (tps > max_tiles) tps = max_tiles;
    int64_t splits = (max_tiles + tps - 1) / tps;
    if (splits > kMaxSplits) {
        splits = kMaxSplits;
        tps = (max_tiles + splits - 1) / splits;
    }
    return Split{static_cast<int>(splits), static_cast<int>(tps)};
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

size_t smem_bytes(int SQ)
{
    return 1024 + kStages * kStage + 2 * kChunk + (SQ * kDq + SQ * kTile + 16 * SQ + 16) * 4 + kNumBars * 8 + 16;
}

std::mutex g_attr_mutex;
bool g_attr_set[64][2];

template <int SQ>
mla_status_t launch(const CUtensorMap &kv, const CUtensorMap &wk, const CUtensorMap &wv, const Params &prm, int grid,
                    cudaStream_t st)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return host::cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= 64) return host::cuda_fail(cudaErrorInvalidDevice, "device index");
    int major = 0;
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e != cudaSuccess) return host::cuda_fail(e, "cudaDeviceGetAttribute(cc)");
    if (major != 10) {
        snprintf(host::g_last_error, sizeof host::g_last_error, "device %d is not sm_100 (compute capability %d.x)",
                 dev, major);
        return MLA_ERR_CUDA;
    }
    const size_t smem = smem_bytes(SQ);
    {
        std::lock_guard<std::mutex> lock(g_attr_mutex);
        if (!g_attr_set[dev][SQ - 1]) {
            e = cudaFuncSetAttribute(mla_naive_kernel<SQ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(smem));
            if (e != cudaSuccess) return host::cuda_fail(e, "cudaFuncSetAttribute(naive)");
            g_attr_set[dev][SQ - 1] = true;
        }
    }
    mla_naive_kernel<SQ><<<grid, kThreads, smem, st>>>(kv, wk, wv, prm);
    e = cudaGetLastError();
    if (e != cudaSuccess) return host::cuda_fail(e, "mla_naive_kernel launch");
    return MLA_OK;
}

}  // namespace naive
}  // namespace mla

using namespace mla;

extern "C" {

size_t mla_decode_naive_workspace_size(int B, int s_q, int H, int max_blocks, int num_sms)
{
    if (B < 1 || B > 4096 || (s_q != 1 && s_q != 2) || H < 1 || H > 128 || max_blocks < 1 || num_sms < 1)
        return 0;
    const naive::Split sp = naive::split_for(B, H, max_blocks, num_sms);
    const size_t pieces = static_cast<size_t>(B) * H * sp.splits;
    return naive::align256(pieces * s_q * naive::kE * sizeof(float)) + naive::align256(pieces * s_q * sizeof(float));
}

mla_status_t mla_decode_naive(const uint16_t *q, const uint16_t *kv_cache, const uint16_t *w_uk,
                              const uint16_t *w_uv, const int32_t *block_table, const int32_t *cache_seqlens,
                              int B, int s_q, int H, int64_t num_blocks, int max_blocks, float softmax_scale,
                              int num_sms, void *workspace, size_t workspace_bytes, int32_t *error_word,
                              uint16_t *out, float *lse, void *stream)
{
    host::clear_error();
    if (!q || !kv_cache || !w_uk || !w_uv || !block_table || !cache_seqlens || !workspace || !error_word || !out ||
        !lse)
        return MLA_ERR_INVALID_ARG;
    if (B < 1 || B > 4096 || H < 1 || H > 128 || num_blocks < 1 || num_blocks > INT32_MAX || max_blocks < 1 ||
        num_sms < 1 || !std::isfinite(softmax_scale))
        return MLA_ERR_INVALID_ARG;
    if (s_q != 1 && s_q != 2) return MLA_ERR_UNSUPPORTED_SHAPE;
    if ((reinterpret_cast<uintptr_t>(q) & 1) || (reinterpret_cast<uintptr_t>(kv_cache) & 15) ||
        (reinterpret_cast<uintptr_t>(w_uk) & 15) || (reinterpret_cast<uintptr_t>(w_uv) & 15) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255) || (reinterpret_cast<uintptr_t>(out) & 7) ||
        (reinterpret_cast<uintptr_t>(lse) & 3) || (reinterpret_cast<uintptr_t>(block_table) & 3) ||
        (reinterpret_cast<uintptr_t>(cache_seqlens) & 3) || (reinterpret_cast<uintptr_t>(error_word) & 3))
        return MLA_ERR_MISALIGNED;
    const size_t need = mla_decode_naive_workspace_size(B, s_q, H, max_blocks, num_sms);
    if (workspace_bytes < need) return MLA_ERR_WORKSPACE_TOO_SMALL;
    const naive::Split sp = naive::split_for(B, H, max_blocks, num_sms);
    const int64_t grid = static_cast<int64_t>(B) * H * sp.splits;
    if (grid > INT32_MAX) return MLA_ERR_INVALID_ARG;

    CUtensorMap kv_map, wk_map, wv_map;
    {
        // the latent cache as [num_blocks][64 rows][576 cols]; box 64 cols x 64 rows x 1 block
        const cuuint64_t dims[3] = {static_cast<cuuint64_t>(MLA_D_QK), static_cast<cuuint64_t>(MLA_PAGE),
                                    static_cast<cuuint64_t>(num_blocks)};
        const cuuint64_t strides[2] = {static_cast<cuuint64_t>(MLA_D_QK) * 2,
                                       static_cast<cuuint64_t>(MLA_PAGE) * MLA_D_QK * 2};
        const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(MLA_PAGE), 1};
        if (!host::tensor_map(&kv_map, "kv", CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, kv_cache, dims, strides, box,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B))
            return MLA_ERR_CUDA;
    }
    {
        // each up-projection as [H * 128 rows][512 cols]; box 64 cols x 128 rows (one head's chunk)
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(MLA_D_V), static_cast<cuuint64_t>(H) * naive::kE};
        const cuuint64_t strides[1] = {static_cast<cuuint64_t>(MLA_D_V) * 2};
        const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(naive::kE)};
        if (!host::tensor_map(&wk_map, "w_uk", CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w_uk, dims, strides, box,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B) ||
            !host::tensor_map(&wv_map, "w_uv", CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w_uv, dims, strides, box,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B))
            return MLA_ERR_CUDA;
    }
    const size_t pieces = static_cast<size_t>(grid);
    naive::Params prm;
    prm.block_table = block_table;
    prm.seqlens = cache_seqlens;
    prm.q = q;
    prm.ws_o = static_cast<float *>(workspace);
    prm.ws_lse = reinterpret_cast<float *>(static_cast<char *>(workspace) +
                                           naive::align256(pieces * s_q * naive::kE * sizeof(float)));
    prm.err = error_word;
    prm.B = B;
    prm.H = H;
    prm.splits = sp.splits;
    prm.tiles_per_split = sp.tiles_per_split;
    prm.max_blocks = max_blocks;
    prm.num_blocks = num_blocks;
    prm.scale = softmax_scale;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const mla_status_t rc = s_q == 1 ? naive::launch<1>(kv_map, wk_map, wv_map, prm, static_cast<int>(grid), st)
                                     : naive::launch<2>(kv_map, wk_map, wv_map, prm, static_cast<int>(grid), st);
    if (rc != MLA_OK) return rc;
    const int64_t rows = static_cast<int64_t>(B) * s_q * H;
    naive::mla_naive_combine_kernel<<<static_cast<unsigned>((rows + 3) / 4), 128, 0, st>>>(
        prm.ws_o, prm.ws_lse, B, s_q, H, sp.splits, out, lse);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return host::cuda_fail(e, "mla_naive_combine_kernel launch");
    return MLA_OK;
}

}  // extern "C"
