/*
 * merge_sm100.cu — merges the result of attention over one block of keys into a running result
 * over other keys: the log-sum-exp merge that Flash-Decoding uses for its key splits, here as a
 * kernel of its own for ring (context-parallel) attention, where the key blocks arrive one after
 * the other from the other ranks.
 *
 * Per row, with the accumulated (o_acc, lse_acc) and the part (o_part, lse_part), natural logs:
 *   M = max(lse_acc, lse_part),  w_a = e^(lse_acc - M),  w_p = e^(lse_part - M)
 *   o_acc <- (w_a o_acc + w_p o_part) / (w_a + w_p),  lse_acc <- M + ln(w_a + w_p)
 * An empty side (lse = -inf: no key yet) gets weight 0; when both are empty the row stays empty.
 *
 * Source (page title, section): "AI Infra 入门：RMSNorm、Softmax、Causal Mask、Sampling 的数学与底层
 * 优化", §3 (LSE paragraph: partial results over key splits combine through their LSEs).
 *
 * One warp per row; lane l owns D/32 consecutive elements (4 for D = 128). The accumulator is fp32
 * so that a chain of merges rounds once, when the bf16 output is written.
 */
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "kernels.h"

namespace attn_b200 {
namespace {

template <int E>  // elements per lane: D / 32
__global__ void __launch_bounds__(256) lse_merge_kernel(float *o_acc, float *lse_acc, const __nv_bfloat16 *o_part,
                                                        const float *lse_part, __nv_bfloat16 *o_out, long long rows)
{
    constexpr int D = 32 * E;
    const int lane = threadIdx.x & 31;
    const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
    for (long long row = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; row < rows;
         row += warps) {
        const float la = lse_acc[row];
        const float lp = lse_part[row];
        const float M = fmaxf(la, lp);
        float wa = 0.f, wp = 0.f;
        if (M != -INFINITY) {  // else both sides are empty
            wa = expf(la - M);  // e^-inf = 0 for an empty side
            wp = expf(lp - M);
        }
        const float sum = wa + wp;
        const float inv = sum > 0.f ? 1.f / sum : 0.f;
        float *acc = o_acc + row * D + lane * E;
        const __nv_bfloat16 *part = o_part + row * D + lane * E;
        float a[E], r[E];
#pragma unroll
        for (int e = 0; e < E; ++e)
            a[e] = acc[e];
#pragma unroll
        for (int e = 0; e < E; ++e)
            r[e] = sum > 0.f ? (wa * a[e] + wp * __bfloat162float(part[e])) * inv : a[e];
#pragma unroll
        for (int e = 0; e < E; ++e)
            acc[e] = r[e];
        if (o_out) {
#pragma unroll
            for (int e = 0; e < E; ++e)
                o_out[row * D + lane * E + e] = __float2bfloat16_rn(r[e]);
        }
        __syncwarp();  // every lane has read lse_acc[row] before it changes
        if (lane == 0)
            lse_acc[row] = sum > 0.f ? M + logf(sum) : M;
    }
}

}  // namespace

cudaError_t launch_lse_merge(float *o_acc, float *lse_acc, const void *o_part, const float *lse_part, void *o_out,
                             long long rows, int D, int sm_count, cudaStream_t stream)
{
    if (rows <= 0)
        return cudaSuccess;
    const long long want = (rows + 7) / 8;  // 8 warps (rows) per block
    const long long cap = static_cast<long long>(sm_count > 0 ? sm_count : 148) * 8;
    const unsigned grid = static_cast<unsigned>(want < cap ? want : cap);
    const auto *part = static_cast<const __nv_bfloat16 *>(o_part);
    auto *out = static_cast<__nv_bfloat16 *>(o_out);
    switch (D) {
    case 32:
        lse_merge_kernel<1><<<grid, 256, 0, stream>>>(o_acc, lse_acc, part, lse_part, out, rows);
        break;
    case 64:
        lse_merge_kernel<2><<<grid, 256, 0, stream>>>(o_acc, lse_acc, part, lse_part, out, rows);
        break;
    case 128:
        lse_merge_kernel<4><<<grid, 256, 0, stream>>>(o_acc, lse_acc, part, lse_part, out, rows);
        break;
    default:
        return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace attn_b200
