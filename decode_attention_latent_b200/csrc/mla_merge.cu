// mla_merge.cu -- merge of partial attention states (context-parallel decode).
//
// W ranks each hold a contiguous range of every sequence's pages and run the
// decode on it; their (out, lse) pairs are merged here through the
// log-sum-exps, the online softmax of "FlashMLA: compressing the KV cache"
// (jsqmd.com), "compute flow", step 4, applied to whole partial results:
//     M = max_w lse_w,  lse = M + ln sum_w exp(lse_w - M),
//     out = sum_w exp(lse_w - lse) out_w.
// The operation is a short streaming pass (W x 1 KB in, 1 KB out per row), so
// it is laid out for coalescing, not for the tensor cores: one warp per row,
// each lane owning 16 of the 512 latent dims (two 16-byte loads per state).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>

#include "mla_decode.h"

namespace mla {
namespace host {
extern thread_local char g_last_error[256];
mla_status_t cuda_fail(cudaError_t e, const char *what);
void clear_error();
}  // namespace host

constexpr int kMergeMaxW = 64;
constexpr int kMergeRowsPerBlock = 4;  // one warp per row
constexpr int kDimsPerLane = 16;       // 512 / 32

__device__ __forceinline__ float2 unpack_bf16x2(uint32_t u)
{
    __nv_bfloat162 h;
    memcpy(&h, &u, sizeof h);
    return __bfloat1622float2(h);
}

__device__ __forceinline__ uint32_t pack_bf16x2_rn(float lo, float hi)
{
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    uint32_t u;
    memcpy(&u, &h, sizeof u);
    return u;
}

__global__ void __launch_bounds__(32 * kMergeRowsPerBlock)
mla_merge_states_kernel(const uint4 *__restrict__ parts, const float *__restrict__ lse_parts, int W, int64_t rows,
                        uint4 *__restrict__ out, float *__restrict__ lse)
{
    const int lane = threadIdx.x & 31;
    const int64_t r = static_cast<int64_t>(blockIdx.x) * kMergeRowsPerBlock + (threadIdx.x >> 5);
    if (r >= rows) return;
    // the largest partial lse, then the total; lane w < W reads state w's lse
    const float lw0 = lane < W ? lse_parts[static_cast<int64_t>(lane) * rows + r] : -INFINITY;
    const float lw1 = lane + 32 < W ? lse_parts[static_cast<int64_t>(lane + 32) * rows + r] : -INFINITY;
    float m = fmaxf(lw0, lw1);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    uint4 *dst = out + r * (512 / 8) + 2 * lane;
    if (m == -INFINITY) {  // no state saw a token
        dst[0] = make_uint4(0, 0, 0, 0);
        dst[1] = make_uint4(0, 0, 0, 0);
        if (lane == 0) lse[r] = -INFINITY;
        return;
    }
    float e = (lw0 == -INFINITY ? 0.f : expf(lw0 - m)) + (lw1 == -INFINITY ? 0.f : expf(lw1 - m));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) e += __shfl_xor_sync(0xffffffffu, e, o);
    const float total = m + logf(e);
    float acc[kDimsPerLane];
#pragma unroll
    for (int k = 0; k < kDimsPerLane; ++k) acc[k] = 0.f;
    for (int w = 0; w < W; ++w) {
        const float l = __shfl_sync(0xffffffffu, w < 32 ? lw0 : lw1, w & 31);
        if (l == -INFINITY) continue;  // uniform across the warp
        const float wt = expf(l - total);
        const uint4 *src = parts + (static_cast<int64_t>(w) * rows + r) * (512 / 8) + 2 * lane;
        const uint4 a = src[0], b = src[1];
        const uint32_t v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const float2 f = unpack_bf16x2(v[k]);
            acc[2 * k] = fmaf(wt, f.x, acc[2 * k]);
            acc[2 * k + 1] = fmaf(wt, f.y, acc[2 * k + 1]);
        }
    }
    dst[0] = make_uint4(pack_bf16x2_rn(acc[0], acc[1]), pack_bf16x2_rn(acc[2], acc[3]),
                        pack_bf16x2_rn(acc[4], acc[5]), pack_bf16x2_rn(acc[6], acc[7]));
    dst[1] = make_uint4(pack_bf16x2_rn(acc[8], acc[9]), pack_bf16x2_rn(acc[10], acc[11]),
                        pack_bf16x2_rn(acc[12], acc[13]), pack_bf16x2_rn(acc[14], acc[15]));
    if (lane == 0) lse[r] = total;
}
}  // namespace mla

extern "C" mla_status_t mla_merge_states(const uint16_t *out_parts, const float *lse_parts, int W, int64_t rows,
                                         uint16_t *out, float *lse, void *stream)
{
    using namespace mla;
    host::clear_error();
    if (!out_parts || !lse_parts || !out || !lse) return MLA_ERR_INVALID_ARG;
    if (W < 1 || W > kMergeMaxW || rows < 1 || rows > INT32_MAX) return MLA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(out_parts) | reinterpret_cast<uintptr_t>(out)) & 15) return MLA_ERR_MISALIGNED;
    if ((reinterpret_cast<uintptr_t>(lse_parts) | reinterpret_cast<uintptr_t>(lse)) & 3) return MLA_ERR_MISALIGNED;
    const int64_t blocks = (rows + kMergeRowsPerBlock - 1) / kMergeRowsPerBlock;
    mla_merge_states_kernel<<<static_cast<unsigned>(blocks), 32 * kMergeRowsPerBlock, 0,
                              static_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<const uint4 *>(out_parts), lse_parts, W, rows, reinterpret_cast<uint4 *>(out), lse);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return host::cuda_fail(e, "mla_merge_states_kernel launch");
    return MLA_OK;
}
