/*
 * decode_sm100.cu — attention of one new query token per (batch, query head) over a bf16 K/V cache
 * (Sq == 1) on sm_100a: split-KV with an LSE merge fused into the same launch.
 *
 * Work split: the Skv cached keys of each (batch, kv head) are cut into `splits` ranges; one CTA
 * handles one range for the G query heads that share the kv head, so each K/V byte is read from
 * HBM once for all of them. A producer warp streams the range through a shared-memory ring with
 * plain bulk copies (one for the K rows, one for the V rows of each stage); four compute warps
 * consume it:
 *
 *   scores   lane l owns D/32 consecutive dims; each warp takes KB = 32/G keys at a time, forms
 *            the G*KB partial dot products and reduces them across the warp with a transposing
 *            butterfly (31 shuffles for 32 sums) that leaves lane l holding score (head l/KB,
 *            key l%KB);
 *   softmax  running max and running sum per head, with the exp(m_old - m_new) rescale of the sum
 *            and of the fp32 accumulator;
 *   PV       each lane accumulates its dims of sum_j p_j v_j for all G heads.
 *
 * The four warps' states are merged in shared memory into the CTA's partial (O_s, LSE_s). With one
 * split that is the answer. Otherwise the partials go to the library workspace and the last CTA
 * to finish a (batch, kv head) — found with an atomic counter, so no CTA ever waits on another —
 * merges them: M = max_s LSE_s, LSE = M + log2 sum_s 2^(LSE_s - M), O = sum_s 2^(LSE_s - LSE) O_s.
 *
 * Sources (page title, section): decode attends to every cached key, no mask needed — "AI Infra
 * 入门：RMSNorm、Softmax、Causal Mask、Sampling 的数学与底层优化", §3; Flash-Decoding split-K merged by
 * LSE — same page, §3 (LSE paragraph); grouped query heads sharing a K/V head and decode being
 * bound by reading K/V (~4 FLOP per byte) — "05 · Tích vô hướng, Softmax và toán của Attention",
 * §4; running max/sum with rescale — same page §6 and "Bộ 06 · Bên trong model", Q1.
 */
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "kernels.h"
#include "sm100_ptx.cuh"

namespace attn_b200 {
namespace {

constexpr int kComputeWarps = 4;
constexpr int kThreads = (kComputeWarps + 1) * 32;  // + one producer warp
constexpr int kStages = 3;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <int D, int G>
struct DecCfg {
    static constexpr int kDPL = D / 32;                 // dims per lane
    static constexpr int kKB = 32 / G;                  // keys per warp batch
    static constexpr int kCK = (kComputeWarps * kKB > 64) ? kComputeWarps * kKB : 64;  // keys per stage
    static constexpr int kBatches = kCK / kKB;          // batches per stage
    static constexpr int kRowBytes = D * 2;
    static constexpr int kStageBytes = 2 * kCK * kRowBytes;  // K rows then V rows
    static constexpr int kOffRing = 0;
    static constexpr int kOffRedO = kOffRing + kStages * kStageBytes;
    static constexpr int kOffRedM = kOffRedO + kComputeWarps * G * D * 4;
    static constexpr int kOffRedL = kOffRedM + kComputeWarps * G * 4;
    static constexpr int kOffBar = ((kOffRedL + kComputeWarps * G * 4 + 15) / 16) * 16;
    static constexpr int kOffFlag = kOffBar + 2 * kStages * 8;
    static constexpr int kSmem = kOffFlag + 16;
};

struct Params {
    const __nv_bfloat16 *q, *k, *v;
    __nv_bfloat16 *o;
    float *lse;
    float *ws_o, *ws_lse;
    int *counters, *status;
    int B, Hq, Hkv, Skv, group, head_groups, splits, chunks_per_split;
    float scale_log2;
};

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void named_sync_compute()
{
    asm volatile("bar.sync 1, %0;" ::"n"(kComputeWarps * 32) : "memory");
}

// Load this lane's kDPL bf16 values of one shared-memory row and widen them to fp32.
template <int DPL>
__device__ __forceinline__ void load_row(const uint8_t *row, int lane, float (&out)[DPL])
{
    if constexpr (DPL == 4) {
        const uint2 w = *reinterpret_cast<const uint2 *>(row + lane * 8);
        out[0] = __uint_as_float(w.x << 16);
        out[1] = __uint_as_float(w.x & 0xffff0000u);
        out[2] = __uint_as_float(w.y << 16);
        out[3] = __uint_as_float(w.y & 0xffff0000u);
    } else if constexpr (DPL == 2) {
        const uint32_t w = *reinterpret_cast<const uint32_t *>(row + lane * 4);
        out[0] = __uint_as_float(w << 16);
        out[1] = __uint_as_float(w & 0xffff0000u);
    } else {
        const uint16_t w = *reinterpret_cast<const uint16_t *>(row + lane * 2);
        out[0] = __uint_as_float(static_cast<uint32_t>(w) << 16);
    }
}

template <int D, int G>
__global__ void __launch_bounds__(kThreads) decode_kernel(const Params p)
{
    using C = DecCfg<D, G>;
    constexpr int DPL = C::kDPL;
    constexpr int KB = C::kKB;
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t s_base = smem_u32(smem);
    float *red_o = reinterpret_cast<float *>(smem + C::kOffRedO);
    float *red_m = reinterpret_cast<float *>(smem + C::kOffRedM);
    float *red_l = reinterpret_cast<float *>(smem + C::kOffRedL);
    const uint32_t bar_full0 = s_base + C::kOffBar;
    const uint32_t bar_empty0 = bar_full0 + 8 * kStages;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::kOffFlag);
    int *last_flag = reinterpret_cast<int *>(smem + C::kOffFlag + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // blockIdx.x = (pair) * splits + split, pair = (b * Hkv + kvh) * head_groups + hg
    const int split = blockIdx.x % p.splits;
    const int pair = blockIdx.x / p.splits;
    const int hg = pair % p.head_groups;
    const int kvh = (pair / p.head_groups) % p.Hkv;
    const int b = pair / (p.head_groups * p.Hkv);
    const int h0 = kvh * p.group + hg * G;  // first query head of this CTA

    const int key_begin = split * p.chunks_per_split * C::kCK;
    const int key_end = min(p.Skv, key_begin + p.chunks_per_split * C::kCK);
    const int n_chunks = (key_end - key_begin + C::kCK - 1) / C::kCK;
    const size_t kv_base = (static_cast<size_t>(b) * p.Hkv + kvh) * static_cast<size_t>(p.Skv) * D;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar_full0 + 8 * s, 1);
            mbar_init(bar_empty0 + 8 * s, kComputeWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kComputeWarps) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int issued = 0;
            for (int c = 0; c < n_chunks; ++c) {
                const int slot = c % kStages;
                const uint32_t round = static_cast<uint32_t>(c / kStages);
                if (!mbar_wait(bar_empty0 + 8 * slot, (round & 1u) ^ 1u, abort_flag, p.status, kSiteDecodeProducer))
                    break;
                const int k0 = key_begin + c * C::kCK;
                const int rows = min(C::kCK, key_end - k0);
                const uint32_t bytes = static_cast<uint32_t>(rows) * C::kRowBytes;
                const uint32_t dst = s_base + C::kOffRing + slot * C::kStageBytes;
                mbar_arrive_expect_tx(bar_full0 + 8 * slot, 2 * bytes);
                bulk_load(dst, p.k + kv_base + static_cast<size_t>(k0) * D, bytes, bar_full0 + 8 * slot);
                bulk_load(dst + C::kCK * C::kRowBytes, p.v + kv_base + static_cast<size_t>(k0) * D, bytes,
                          bar_full0 + 8 * slot);
                ++issued;
            }
            if (*abort_flag) {
                for (int c = (issued > kStages ? issued - kStages : 0); c < issued; ++c) {
                    const uint32_t bar = bar_full0 + 8 * (c % kStages);
                    const uint32_t par = static_cast<uint32_t>(c / kStages) & 1u;
                    const uint64_t t0 = global_timer_ns();
                    while (!mbar_try_wait(bar, par) && global_timer_ns() - t0 < 100000000ull) {
                    }
                }
            }
        }
        return;  // the producer takes no part in the merge below
    }

    // ---------------------------------------------------------------- compute warps
    float q[G][DPL];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const __nv_bfloat16 *qrow = p.q + (static_cast<size_t>(b) * p.Hq + h0 + g) * D + lane * DPL;
#pragma unroll
        for (int i = 0; i < DPL; ++i)
            q[g][i] = __bfloat162float(qrow[i]);
    }
    float acc[G][DPL];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int i = 0; i < DPL; ++i)
            acc[g][i] = 0.f;
    float m_run = -INFINITY;  // running max of head (lane / KB), log2-scaled units
    float lsum = 0.f;          // this lane's share of that head's running sum
    const int my_key = lane % KB;

    bool ok = true;
    for (int c = 0; c < n_chunks; ++c) {
        const int slot = c % kStages;
        if (!(ok = mbar_wait(bar_full0 + 8 * slot, static_cast<uint32_t>(c / kStages) & 1u, abort_flag, p.status,
                             kSiteDecodeConsumer)))
            break;
        const int rows = min(C::kCK, key_end - (key_begin + c * C::kCK));
        const uint8_t *sk = smem + C::kOffRing + slot * C::kStageBytes;
        const uint8_t *sv = sk + C::kCK * C::kRowBytes;

        for (int bt = warp; bt < C::kBatches; bt += kComputeWarps) {
            const int key0 = bt * KB;
            if (key0 >= rows)
                break;
            // partial dot products: part[g * KB + kk] over this lane's dims
            float part[32];
#pragma unroll
            for (int kk = 0; kk < KB; ++kk) {
                float kv[DPL];
                load_row<DPL>(sk + (key0 + kk) * C::kRowBytes, lane, kv);
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    float s = 0.f;
#pragma unroll
                    for (int i = 0; i < DPL; ++i)
                        s = fmaf(q[g][i], kv[i], s);
                    part[g * KB + kk] = s;
                }
            }
            // transposing butterfly: after the step with offset s a lane keeps the half of its
            // current block selected by (lane & s); at the end lane l holds the total of index l.
#pragma unroll
            for (int s = 16; s >= 1; s >>= 1) {
                const bool upper = (lane & s) != 0;
#pragma unroll
                for (int i = 0; i < s; ++i) {
                    const float send = upper ? part[i] : part[i + s];
                    const float keep = upper ? part[i + s] : part[i];
                    part[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
                }
            }
            const bool valid = key0 + my_key < rows;
            const float s2 = valid ? part[0] * p.scale_log2 : -INFINITY;
            float mx = s2;
#pragma unroll
            for (int o = 1; o < KB; o <<= 1)
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            const float m_new = fmaxf(m_run, mx);  // finite: key0 < rows, so each head sees a key
            const float alpha = ex2(m_run - m_new);
            const float pv = ex2(s2 - m_new);
            lsum = lsum * alpha + pv;
            m_run = m_new;
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float a = __shfl_sync(0xffffffffu, alpha, g * KB);
#pragma unroll
                for (int i = 0; i < DPL; ++i)
                    acc[g][i] *= a;
            }
#pragma unroll
            for (int kk = 0; kk < KB; ++kk) {
                if (key0 + kk >= rows)
                    break;  // uniform across the warp; stale rows past the range are never read
                float vv[DPL];
                load_row<DPL>(sv + (key0 + kk) * C::kRowBytes, lane, vv);
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float w = __shfl_sync(0xffffffffu, pv, g * KB + kk);
#pragma unroll
                    for (int i = 0; i < DPL; ++i)
                        acc[g][i] = fmaf(w, vv[i], acc[g][i]);
                }
            }
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(bar_empty0 + 8 * slot);
    }

    // ---------------------------------------------------------------- merge the four warps
#pragma unroll
    for (int o = 1; o < KB; o <<= 1)
        lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
    if (my_key == 0 && lane / KB < G) {
        red_m[warp * G + lane / KB] = m_run;
        red_l[warp * G + lane / KB] = lsum;
    }
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int i = 0; i < DPL; ++i)
            red_o[(warp * G + g) * D + lane * DPL + i] = acc[g][i];
    named_sync_compute();

    const int tid = threadIdx.x;  // 0 .. 127
    const int n_out = G * D;
    for (int idx = tid; idx < n_out; idx += kComputeWarps * 32) {
        const int g = idx / D;
        const int d = idx % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kComputeWarps; ++w)
            M = fmaxf(M, red_m[w * G + g]);
        float L = 0.f, O = 0.f;
#pragma unroll
        for (int w = 0; w < kComputeWarps; ++w) {
            const float mw = red_m[w * G + g];
            const float e = (mw == -INFINITY) ? 0.f : ex2(mw - M);
            L = fmaf(red_l[w * G + g], e, L);
            O = fmaf(red_o[(w * G + g) * D + d], e, O);
        }
        const size_t bh = static_cast<size_t>(b) * p.Hq + h0 + g;
        if (p.splits == 1) {
            p.o[bh * D + d] = __float2bfloat16_rn(O / L);
            if (d == 0)
                p.lse[bh] = (M + log2f(L)) * kLn2;
        } else {
            p.ws_o[(bh * p.splits + split) * D + d] = O / L;
            if (d == 0)
                p.ws_lse[bh * p.splits + split] = M + log2f(L);
        }
    }
    if (p.splits == 1)
        return;

    // ---------------------------------------------------------------- last CTA of the pair merges the splits
    __threadfence();
    named_sync_compute();
    if (tid == 0) {
        const int prev = atomicAdd(&p.counters[pair], 1);
        *last_flag = (prev == p.splits - 1) ? 1 : 0;
    }
    named_sync_compute();
    if (!*last_flag)
        return;
    __threadfence();
    for (int idx = tid; idx < n_out; idx += kComputeWarps * 32) {
        const int g = idx / D;
        const int d = idx % D;
        const size_t bh = static_cast<size_t>(b) * p.Hq + h0 + g;
        const float *lse_s = p.ws_lse + bh * p.splits;
        float M = -INFINITY;
        for (int s = 0; s < p.splits; ++s)
            M = fmaxf(M, __ldcg(lse_s + s));
        float W = 0.f, O = 0.f;
        for (int s = 0; s < p.splits; ++s) {
            const float w = ex2(__ldcg(lse_s + s) - M);
            W += w;
            O = fmaf(w, __ldcg(p.ws_o + (bh * p.splits + s) * D + d), O);
        }
        p.o[bh * D + d] = __float2bfloat16_rn(O / W);
        if (d == 0)
            p.lse[bh] = (M + log2f(W)) * kLn2;
    }
    if (tid == 0)
        atomicExch(&p.counters[pair], 0);  // ready for the next call
}

template <int D, int G>
cudaError_t launch_dg(const DecodeArgs &a, cudaStream_t stream)
{
    using C = DecCfg<D, G>;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(decode_kernel<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
        if (e != cudaSuccess)
            return e;
        attr_set = true;
    }
    Params p;
    p.q = static_cast<const __nv_bfloat16 *>(a.q);
    p.k = static_cast<const __nv_bfloat16 *>(a.k);
    p.v = static_cast<const __nv_bfloat16 *>(a.v);
    p.o = static_cast<__nv_bfloat16 *>(a.o);
    p.lse = a.lse;
    p.ws_o = a.ws_o;
    p.ws_lse = a.ws_lse;
    p.counters = a.counters;
    p.status = a.status;
    p.B = a.B;
    p.Hq = a.Hq;
    p.Hkv = a.Hkv;
    p.Skv = a.Skv;
    p.group = a.Hq / a.Hkv;
    p.head_groups = p.group / G;
    p.splits = a.splits;
    const int n_chunks = (a.Skv + C::kCK - 1) / C::kCK;
    p.chunks_per_split = (n_chunks + a.splits - 1) / a.splits;
    p.scale_log2 = a.scale * kLog2e;
    const long long grid = static_cast<long long>(a.B) * a.Hkv * p.head_groups * a.splits;
    decode_kernel<D, G><<<static_cast<unsigned>(grid), kThreads, C::kSmem, stream>>>(p);
    return cudaGetLastError();
}

template <int D, int G>
int occupancy_dg()
{
    using C = DecCfg<D, G>;
    static int cached = 0;
    if (cached == 0) {
        int n = 0;
        if (cudaFuncSetAttribute(decode_kernel<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem) !=
                cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_kernel<D, G>, kThreads, C::kSmem) != cudaSuccess)
            n = 1;
        cached = n > 0 ? n : 1;
    }
    return cached;
}

template <int D>
cudaError_t launch_d(const DecodeArgs &a, cudaStream_t stream)
{
    switch (decode_heads_per_cta(a.Hq / a.Hkv)) {
    case 1:
        return launch_dg<D, 1>(a, stream);
    case 2:
        return launch_dg<D, 2>(a, stream);
    case 4:
        return launch_dg<D, 4>(a, stream);
    default:
        return launch_dg<D, 8>(a, stream);
    }
}

template <int D>
int occupancy_d(int group)
{
    switch (decode_heads_per_cta(group)) {
    case 1:
        return occupancy_dg<D, 1>();
    case 2:
        return occupancy_dg<D, 2>();
    case 4:
        return occupancy_dg<D, 4>();
    default:
        return occupancy_dg<D, 8>();
    }
}

}  // namespace

int decode_heads_per_cta(int group)
{
    // Largest power of two <= 8 that divides the group size.
    if (group % 8 == 0)
        return 8;
    if (group % 4 == 0)
        return 4;
    if (group % 2 == 0)
        return 2;
    return 1;
}

int decode_keys_per_chunk(int group)
{
    const int kb = 32 / decode_heads_per_cta(group);
    return (kComputeWarps * kb > 64) ? kComputeWarps * kb : 64;
}

int decode_effective_splits(int Skv, int group, int requested)
{
    const int ck = decode_keys_per_chunk(group);
    const int n_chunks = (Skv + ck - 1) / ck;
    int s = requested < 1 ? 1 : requested;
    if (s > n_chunks)
        s = n_chunks;
    const int per = (n_chunks + s - 1) / s;
    return (n_chunks + per - 1) / per;  // every split starts inside the key range
}

int decode_ctas_per_sm(int D, int group)
{
    switch (D) {
    case 32:
        return occupancy_d<32>(group);
    case 64:
        return occupancy_d<64>(group);
    default:
        return occupancy_d<128>(group);
    }
}

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream)
{
    switch (a.D) {
    case 32:
        return launch_d<32>(a, stream);
    case 64:
        return launch_d<64>(a, stream);
    case 128:
        return launch_d<128>(a, stream);
    default:
        return cudaErrorInvalidValue;
    }
}

}  // namespace attn_b200
