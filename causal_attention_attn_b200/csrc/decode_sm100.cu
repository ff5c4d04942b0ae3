/*
 * decode_sm100.cu — attention of one new query token per (batch, query head) over a bf16 K/V cache
 * (Sq == 1) on sm_100a for head dims 32 and 64 (head dim 128 runs on the tensor core,
 * decode_tc_sm100.cu): a persistent split-KV kernel with the LSE merge fused into the same launch.
 * This file also holds the decode plan both kernels share.
 *
 * Work: a "pair" is one (batch, kv head, group of G query heads sharing that kv head); its Skv keys
 * are cut into chunks of CK keys. All pairs' chunks form one sequence of T = pairs * chunks_per_pair
 * units, and CTA c of the P launched CTAs takes the contiguous range [c*T/P, (c+1)*T/P) — as many
 * CTAs as fit on the GPU at once, each with the same amount of K/V to read, so the work is balanced
 * whatever B, Hkv and Skv are. A range may cover the end of one pair and the start of the next: each
 * piece ("segment") yields either the pair's final output (when the CTA holds the whole pair) or a
 * partial (O_s, LSE_s); once its range is streamed, a CTA signals the shared pairs it contributed
 * to, and the last CTA to finish a shared pair — found with an atomic counter, so no CTA ever waits
 * on another — merges the partials: M = max_s LSE_s,
 * LSE = M + log2 sum_s 2^(LSE_s - M), O = sum_s 2^(LSE_s - LSE) O_s.
 *
 * Inside a CTA a producer warp streams the range's chunks (K rows, then V rows, plain bulk copies)
 * through a shared-memory ring, together with each segment's q rows; seven compute warps consume
 * it (one CTA per SM). The eight lanes of a "lane group" share one key row; lane t of the group owns
 * D/8 of the dims (for D = 128: dims 8t..8t+7 and 64+8t..64+8t+7, two conflict-free 16-byte loads
 * per row) and keeps q and its slice of the O accumulator of all G heads in registers. A group takes
 * 8/G keys at a time:
 *
 *   scores   G*(8/G) = 8 partial dot products per lane (packed f32x2 FMAs), reduced across the
 *            group by a transposing butterfly (7 shuffles for 8 sums) that leaves lane t with
 *            score (head t/(8/G), key t%(8/G));
 *   softmax  running (reference) max and running sum per head and group, with the
 *            exp(m_old - m_new) rescale of the sum and of the fp32 accumulator when the max grows
 *            by more than 2^8;
 *   PV       each lane accumulates its dims of sum_j p_j v_j for all G heads (f32x2 FMAs).
 *
 * At the end of a segment the groups merge by shuffles, the warps through shared memory.
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
#include <type_traits>

#include "kernels.h"
#include "sm100_ptx.cuh"

namespace attn_b200 {
namespace {

#ifndef ATTN_DECODE_STAGES
#define ATTN_DECODE_STAGES 3
#endif
#ifndef ATTN_DECODE_MIN_CHUNK
#define ATTN_DECODE_MIN_CHUNK 64
#endif
constexpr int kMaxStages = ATTN_DECODE_STAGES;  // K/V chunks in flight per CTA, when they fit
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;

#ifndef ATTN_DECODE_LANES
#define ATTN_DECODE_LANES 8
#endif

// Lanes that share one key row (a "lane group"): eight. (Sixteen-lane groups, which halve each
// thread's registers and fit eleven compute warps, measured slower: more shuffles per key.)
__host__ __device__ constexpr int lanes_per_key(int G) { return G == 1 ? 8 : ATTN_DECODE_LANES; }
// Compute warps per CTA (plus the producer warp; one CTA per SM). With 16-lane groups each thread
// holds half as much q and accumulator, so three warps fit per SM sub-partition.
__host__ __device__ constexpr int compute_warps(int G)
{
    return lanes_per_key(G) == 16 ? 11 : (G == 1 ? 4 : 7);
}
__host__ __device__ constexpr int keys_per_group_batch(int G) { return lanes_per_key(G) / G; }
__host__ __device__ constexpr int keys_per_round(int G)
{
    return compute_warps(G) * (32 / lanes_per_key(G)) * keys_per_group_batch(G);
}
// Keys per chunk: whole rounds of all groups' batches, at least ATTN_DECODE_MIN_CHUNK keys.
__host__ __device__ constexpr int keys_per_stage(int G)
{
    return ((ATTN_DECODE_MIN_CHUNK + keys_per_round(G) - 1) / keys_per_round(G)) * keys_per_round(G);
}

template <int D, int G>
struct DecCfg {
    static constexpr int kLG = lanes_per_key(G);           // lanes per key row
    static constexpr int kComputeWarps = compute_warps(G);
    static constexpr int kGroups = kComputeWarps * (32 / kLG);
    static constexpr int kThreads = (kComputeWarps + 1) * 32;  // + one producer warp
    static constexpr int kDPL = D / kLG;                  // dims per lane
    static constexpr int kKB = keys_per_group_batch(G);   // keys per group batch
    static constexpr int kCK = keys_per_stage(G);         // keys per chunk (pipeline stage)
    static constexpr int kRowBytes = D * 2;
    static constexpr int kStageBytes = 2 * kCK * kRowBytes;  // K rows then V rows
    static constexpr int kStages = (kMaxStages * kStageBytes <= 190 * 1024) ? kMaxStages
                                   : ((190 * 1024 / kStageBytes) >= 2 ? 190 * 1024 / kStageBytes : 2);
    static constexpr int kQBytes = G * D * 2;                // one segment's q rows
    static constexpr int kQSlot = ((kQBytes + 127) / 128) * 128;
    static constexpr int kOffRing = 0;
    static constexpr int kOffQ = kOffRing + kStages * kStageBytes;
    static constexpr int kOffRedO = kOffQ + 2 * kQSlot;
    static constexpr int kOffRedM = kOffRedO + kComputeWarps * G * D * 4;
    static constexpr int kOffRedL = kOffRedM + kComputeWarps * G * 4;
    static constexpr int kOffBar = ((kOffRedL + kComputeWarps * G * 4 + 15) / 16) * 16;
    static constexpr int kNumBars = 2 * kStages + 4;  // full, empty, q full, q empty
    static constexpr int kOffFlag = kOffBar + kNumBars * 8;
    static constexpr int kSmem = kOffFlag + 32;
    static_assert(G * kKB == kLG, "one score per lane after the butterfly");
    static_assert(kDPL >= 2, "at least one bf16 pair per lane");
    static_assert(kCK % (kGroups * kKB) == 0, "a chunk is whole rounds of group batches");
    static_assert(kSmem <= 227 * 1024, "shared memory budget");
};

struct Params {
    const __nv_bfloat16 *q, *k, *v;
    __nv_bfloat16 *o;
    float *lse;
    float *ws;  // partials: [pairs][max_contrib][G*D + G]
    int *counters, *status;
    int Hq, Hkv, Skv, group, head_groups, cpp, ctas, max_contrib;
    long long total;
    float scale_log2;
};

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

template <int NT>
__device__ __forceinline__ void named_sync_compute()
{
    asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory");
}

// First unit of CTA c's range: floor(c * T / P).
__device__ __forceinline__ long long range_start(long long c, long long total, int ctas)
{
    return c * total / ctas;
}

// The CTA whose range holds unit g: the largest c with range_start(c) <= g (c0 or c0 + 1).
__device__ __forceinline__ int cta_of_unit(long long g, long long total, int ctas)
{
    long long c0 = g * ctas / total;
    if (c0 + 1 < ctas && range_start(c0 + 1, total, ctas) <= g)
        ++c0;
    return static_cast<int>(c0);
}

// bf16x2 word -> (low element, high element) as fp32.
__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t w)
{
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// This lane's D/LG elements of one shared-memory row, as D/(2 LG) packed bf16x2 words.
// LG = 8:  D = 128: bytes [16t, 16t+16) and [128+16t, 128+16t+16); D = 64: [16t, 16t+16); D = 32: [8t, 8t+8).
// LG = 16: one contiguous piece of D/8 bytes at t * D/8 (16, 8 or 4 bytes).
// Within each eight lanes the loads cover 128 (or 64) consecutive bytes: no bank conflicts.
template <int D, int LG>
__device__ __forceinline__ void load_row_words(const uint8_t *row, int t, uint32_t (&w)[D / (2 * LG)])
{
    if constexpr (LG == 8 && D == 128) {
        const uint4 a = *reinterpret_cast<const uint4 *>(row + 16 * t);
        const uint4 b = *reinterpret_cast<const uint4 *>(row + 128 + 16 * t);
        w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
        w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
    } else if constexpr ((LG == 8 && D == 64) || (LG == 16 && D == 128)) {
        const uint4 a = *reinterpret_cast<const uint4 *>(row + 16 * t);
        w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    } else if constexpr ((LG == 8 && D == 32) || (LG == 16 && D == 64)) {
        const uint2 a = *reinterpret_cast<const uint2 *>(row + 8 * t);
        w[0] = a.x; w[1] = a.y;
    } else {
        static_assert(LG == 16 && D == 32, "unsupported lane group");
        w[0] = *reinterpret_cast<const uint32_t *>(row + 4 * t);
    }
}

// Element index (within the row) of this lane's i-th owned dim, matching load_row_words.
template <int D, int LG>
__device__ __forceinline__ int owned_dim(int t, int i)
{
    if constexpr (LG == 8 && D == 128)
        return (i < 8) ? 8 * t + i : 64 + 8 * t + (i - 8);
    else
        return (D / LG) * t + i;
}

template <int D, int G>
__global__ void __launch_bounds__(DecCfg<D, G>::kThreads, 1) decode_kernel(const Params p)
{
    using C = DecCfg<D, G>;
    constexpr int kStages = C::kStages;
    constexpr int kComputeWarps = C::kComputeWarps;
    constexpr int LG = C::kLG;
    constexpr int kGroups = C::kGroups;
    constexpr int NW2 = C::kDPL / 2;  // packed pairs per lane
    constexpr int KB = C::kKB;
    constexpr int CK = C::kCK;
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t s_base = smem_u32(smem);
    float *red_o = reinterpret_cast<float *>(smem + C::kOffRedO);
    float *red_m = reinterpret_cast<float *>(smem + C::kOffRedM);
    float *red_l = reinterpret_cast<float *>(smem + C::kOffRedL);
    const uint32_t bar_full0 = s_base + C::kOffBar;
    const uint32_t bar_empty0 = bar_full0 + 8 * kStages;
    const uint32_t bar_qfull0 = bar_empty0 + 8 * kStages;
    const uint32_t bar_qempty0 = bar_qfull0 + 16;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::kOffFlag);
    int *last_flag = reinterpret_cast<int *>(smem + C::kOffFlag + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int cta = blockIdx.x;
    const long long g_begin = range_start(cta, p.total, p.ctas);
    const long long g_end = range_start(cta + 1, p.total, p.ctas);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar_full0 + 8 * s, 1);
            mbar_init(bar_empty0 + 8 * s, kComputeWarps);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar_qfull0 + 8 * s, 1);
            mbar_init(bar_qempty0 + 8 * s, kComputeWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kComputeWarps) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
#ifdef ATTN_DECODE_EVICT_FIRST
            const uint64_t pol = l2_policy_evict_first();  // every K/V byte is read exactly once
#endif
            int issued = 0, seg = 0;
            // Walk the range with counters instead of dividing the unit index for every chunk.
            long long pair = g_begin / p.cpp;
            int local = static_cast<int>(g_begin - pair * p.cpp);
            const __nv_bfloat16 *kp = nullptr, *vp = nullptr;
            for (long long g = g_begin; g < g_end; ++g) {
                if (g == g_begin || local == 0) {
                    // A new segment: its q rows (G heads, contiguous) into the segment's q slot.
                    const int qs = seg & 1;
                    if (!mbar_wait(bar_qempty0 + 8 * qs, (static_cast<uint32_t>(seg >> 1) & 1u) ^ 1u, abort_flag,
                                   p.status, kSiteDecodeProducer))
                        break;
                    const int hg = static_cast<int>(pair % p.head_groups);
                    const long long bk = pair / p.head_groups;  // b * Hkv + kvh
                    const long long b = bk / p.Hkv;
                    const int kvh = static_cast<int>(bk % p.Hkv);
                    const int h0 = kvh * p.group + hg * G;
                    mbar_arrive_expect_tx(bar_qfull0 + 8 * qs, C::kQBytes);
                    bulk_load(s_base + C::kOffQ + qs * C::kQSlot, p.q + (b * p.Hq + h0) * D, C::kQBytes,
                              bar_qfull0 + 8 * qs);
                    kp = p.k + static_cast<size_t>(bk) * p.Skv * D;
                    vp = p.v + static_cast<size_t>(bk) * p.Skv * D;
                    ++seg;
                }
                const int slot = issued % kStages;
                if (!mbar_wait(bar_empty0 + 8 * slot, (static_cast<uint32_t>(issued / kStages) & 1u) ^ 1u, abort_flag,
                               p.status, kSiteDecodeProducer))
                    break;
                const int k0 = local * CK;
                const int rows = min(CK, p.Skv - k0);
                const uint32_t bytes = static_cast<uint32_t>(rows) * C::kRowBytes;
                const uint32_t dst = s_base + C::kOffRing + slot * C::kStageBytes;
                mbar_arrive_expect_tx(bar_full0 + 8 * slot, 2 * bytes);
#ifdef ATTN_DECODE_EVICT_FIRST
                bulk_load_hint(dst, kp + static_cast<size_t>(k0) * D, bytes, bar_full0 + 8 * slot, pol);
                bulk_load_hint(dst + CK * C::kRowBytes, vp + static_cast<size_t>(k0) * D, bytes, bar_full0 + 8 * slot,
                               pol);
#else
                bulk_load(dst, kp + static_cast<size_t>(k0) * D, bytes, bar_full0 + 8 * slot);
                bulk_load(dst + CK * C::kRowBytes, vp + static_cast<size_t>(k0) * D, bytes, bar_full0 + 8 * slot);
#endif
                ++issued;
                if (++local == p.cpp) {
                    local = 0;
                    ++pair;
                }
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
        return;  // the producer takes no part in the merges below
    }

    // ---------------------------------------------------------------- compute warps
    const int t = lane % LG;                             // lane within its group
    const int group_id = warp * (32 / LG) + lane / LG;   // lane group within the CTA
    const int obase = lane & ~(LG - 1);                  // first lane of this group
    const int my_head = t / KB;  // head of the score this lane holds after the butterfly
    const int my_key = t % KB;   // key (within the group batch) of that score
    const int tid = threadIdx.x;            // 0 .. 32 * kComputeWarps - 1
    constexpr int n_out = G * D;
    (void)my_head;

    int consumed = 0, seg = 0;
    bool ok = true;
    // Shared pairs whose partial this CTA wrote (at most the range's first and last segment).
    __shared__ long long deferred_pair[2];
    __shared__ int deferred_first[2];
    int n_deferred = 0;  // meaningful in thread 0 only
    for (long long g = g_begin; ok && g < g_end; ++seg) {
        const long long pair = g / p.cpp;
        const int local0 = static_cast<int>(g - pair * p.cpp);
        const long long seg_end = min(g_end, (pair + 1) * p.cpp);
        const int n_chunks = static_cast<int>(seg_end - g);
        const bool whole_pair = (local0 == 0) && (seg_end == (pair + 1) * p.cpp);
        const long long bk = pair / p.head_groups;
        const long long b = bk / p.Hkv;
        const int kvh = static_cast<int>(bk % p.Hkv);
        const int h0 = kvh * p.group + static_cast<int>(pair % p.head_groups) * G;

        // q of this segment, from its shared-memory slot
        const int qs = seg & 1;
        ok = mbar_wait(bar_qfull0 + 8 * qs, static_cast<uint32_t>(seg >> 1) & 1u, abort_flag, p.status,
                       kSiteDecodeConsumer);
        const __nv_bfloat16 *sq = reinterpret_cast<const __nv_bfloat16 *>(smem + C::kOffQ + qs * C::kQSlot);
        float2 q2[G][NW2];
#pragma unroll
        for (int gg = 0; gg < G; ++gg)
#pragma unroll
            for (int i = 0; i < NW2; ++i)
                q2[gg][i] = make_float2(__bfloat162float(sq[gg * D + owned_dim<D, LG>(t, 2 * i)]) * p.scale_log2,
                                        __bfloat162float(sq[gg * D + owned_dim<D, LG>(t, 2 * i + 1)]) * p.scale_log2);
        __syncwarp();
        if (lane == 0)
            mbar_arrive(bar_qempty0 + 8 * qs);

        float2 acc[G][NW2];
#pragma unroll
        for (int gg = 0; gg < G; ++gg)
#pragma unroll
            for (int i = 0; i < NW2; ++i)
                acc[gg][i] = make_float2(0.f, 0.f);
        float m_run = -INFINITY;  // running max of head my_head in this group, log2-scaled units
        float lsum = 0.f;          // this lane's share of that head's running sum

        for (int ci = 0; ok && ci < n_chunks; ++ci, ++consumed) {
            const int slot = consumed % kStages;
            if (!(ok = mbar_wait(bar_full0 + 8 * slot, static_cast<uint32_t>(consumed / kStages) & 1u, abort_flag,
                                 p.status, kSiteDecodeConsumer)))
                break;
            const int rows = min(CK, p.Skv - (local0 + ci) * CK);
            const uint8_t *sk = smem + C::kOffRing + slot * C::kStageBytes;
            const uint8_t *sv = sk + CK * C::kRowBytes;

            // One batch of KB keys for this lane group, starting at key0. In a full chunk every key is
            // valid; in the ragged last chunk of a pair keys past `rows` are masked (score -inf, V
            // row taken as zero). `full` is a compile-time flag so that the common case carries no
            // bounds checks.
            auto batch = [&](auto full_tag, int key0) {
                constexpr bool kFull = decltype(full_tag)::value;
                uint32_t kw[KB][NW2];
#pragma unroll
                for (int kk = 0; kk < KB; ++kk) {
                    if (kFull || key0 + kk < rows)
                        load_row_words<D, LG>(sk + (key0 + kk) * C::kRowBytes, t, kw[kk]);
                    else
#pragma unroll
                        for (int i = 0; i < NW2; ++i)
                            kw[kk][i] = 0u;
                }
                // Widen each K element once; the G heads then share it.
                float2 kf[KB][NW2];
#pragma unroll
                for (int kk = 0; kk < KB; ++kk)
#pragma unroll
                    for (int i = 0; i < NW2; ++i)
                        kf[kk][i] = bf16x2_to_float2(kw[kk][i]);
                float part[LG];
#pragma unroll
                for (int gg = 0; gg < G; ++gg) {
                    float2 s2[KB];
#pragma unroll
                    for (int kk = 0; kk < KB; ++kk)
                        s2[kk] = make_float2(0.f, 0.f);
#pragma unroll
                    for (int i = 0; i < NW2; ++i) {
#pragma unroll
                        for (int kk = 0; kk < KB; ++kk)
                            s2[kk] = __ffma2_rn(q2[gg][i], kf[kk][i], s2[kk]);
                    }
#pragma unroll
                    for (int kk = 0; kk < KB; ++kk)
                        part[gg * KB + kk] = s2[kk].x + s2[kk].y;
                }
                // Transposing butterfly inside the group: lane t ends with the total of index t.
#pragma unroll
                for (int s = LG / 2; s >= 1; s >>= 1) {
                    const bool upper = (t & s) != 0;
#pragma unroll
                    for (int i = 0; i < s; ++i) {
                        const float send = upper ? part[i] : part[i + s];
                        const float keep = upper ? part[i + s] : part[i];
                        part[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
                    }
                }
                // q was pre-scaled into log2 units, so part[0] is the score in those units.
                const float s2 = (kFull || key0 + my_key < rows) ? part[0] : -INFINITY;
                float mx = s2;
#pragma unroll
                for (int o = 1; o < KB; o <<= 1)
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                // The reference max m_run only moves when the batch max exceeds it by more than 8
                // (log2 units): weights stay below 2^8 and the accumulators are rescaled rarely;
                // O and the sum are both relative to m_run, so O / sum is unchanged. In a ragged
                // chunk a group batch may lie wholly past `rows`: its state is then unchanged.
                const bool move = mx > m_run + kRescaleThreshold;
                const float m_new = move ? mx : m_run;
                const float alpha = move ? ex2(m_run - m_new) : 1.f;
                const float pv = (!kFull && m_new == -INFINITY) ? 0.f : ex2(s2 - m_new);
                lsum = lsum * alpha + pv;
                m_run = m_new;
                if (__any_sync(0xffffffffu, move)) {
#pragma unroll
                    for (int gg = 0; gg < G; ++gg) {
                        const float a = __shfl_sync(0xffffffffu, alpha, obase + gg * KB);
#pragma unroll
                        for (int i = 0; i < NW2; ++i)
                            acc[gg][i] = __fmul2_rn(acc[gg][i], make_float2(a, a));
                    }
                }
#pragma unroll
                for (int kk = 0; kk < KB; ++kk) {
                    uint32_t vw[NW2];
                    if (kFull || key0 + kk < rows)
                        load_row_words<D, LG>(sv + (key0 + kk) * C::kRowBytes, t, vw);
                    else
#pragma unroll
                        for (int i = 0; i < NW2; ++i)
                            vw[i] = 0u;
                    float2 vf[NW2];
#pragma unroll
                    for (int i = 0; i < NW2; ++i)
                        vf[i] = bf16x2_to_float2(vw[i]);
#pragma unroll
                    for (int gg = 0; gg < G; ++gg) {
                        const float w = __shfl_sync(0xffffffffu, pv, obase + gg * KB + kk);
                        const float2 w2 = make_float2(w, w);
#pragma unroll
                        for (int i = 0; i < NW2; ++i)
                            acc[gg][i] = __ffma2_rn(w2, vf[i], acc[gg][i]);
                    }
                }
            };
            constexpr int kRound = kGroups * KB;  // keys covered by one batch of every lane group
            if (rows == CK) {
#pragma unroll
                for (int r = 0; r < CK / kRound; ++r)
                    batch(std::true_type{}, r * kRound + group_id * KB);
            } else {
                // The loop bound is warp-uniform (key0 - group_id * KB is a multiple of kRound).
                for (int key0 = group_id * KB; key0 - group_id * KB < rows; key0 += kRound)
                    batch(std::false_type{}, key0);
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar_empty0 + 8 * slot);
        }

        // ------------------------------------------------ end of segment: merge lane groups, then warps
#pragma unroll
        for (int o = 1; o < KB; o <<= 1)
            lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
        float mg[G], lg[G];
#pragma unroll
        for (int gg = 0; gg < G; ++gg) {
            mg[gg] = __shfl_sync(0xffffffffu, m_run, obase + gg * KB);
            lg[gg] = __shfl_sync(0xffffffffu, lsum, obase + gg * KB);
        }
#pragma unroll
        for (int off = LG; off < 32; off <<= 1) {
#pragma unroll
            for (int gg = 0; gg < G; ++gg) {
                const float m2 = __shfl_xor_sync(0xffffffffu, mg[gg], off);
                const float l2 = __shfl_xor_sync(0xffffffffu, lg[gg], off);
                const float M = fmaxf(mg[gg], m2);
                const float a1 = (mg[gg] == -INFINITY) ? 0.f : ex2(mg[gg] - M);
                const float a2 = (m2 == -INFINITY) ? 0.f : ex2(m2 - M);
                lg[gg] = lg[gg] * a1 + l2 * a2;
                mg[gg] = M;
#pragma unroll
                for (int i = 0; i < NW2; ++i) {
                    const float2 y = make_float2(__shfl_xor_sync(0xffffffffu, acc[gg][i].x, off),
                                                 __shfl_xor_sync(0xffffffffu, acc[gg][i].y, off));
                    acc[gg][i] = __ffma2_rn(acc[gg][i], make_float2(a1, a1), __fmul2_rn(y, make_float2(a2, a2)));
                }
            }
        }
        if (lane < LG) {
#pragma unroll
            for (int gg = 0; gg < G; ++gg) {
#pragma unroll
                for (int i = 0; i < NW2; ++i) {
                    red_o[(warp * G + gg) * D + owned_dim<D, LG>(t, 2 * i)] = acc[gg][i].x;
                    red_o[(warp * G + gg) * D + owned_dim<D, LG>(t, 2 * i + 1)] = acc[gg][i].y;
                }
                if (lane == 0) {
                    red_m[warp * G + gg] = mg[gg];
                    red_l[warp * G + gg] = lg[gg];
                }
            }
        }
        named_sync_compute<kComputeWarps * 32>();

        int contrib_first = 0;
        if (!whole_pair)
            contrib_first = cta_of_unit(pair * p.cpp, p.total, p.ctas);
        float *slot_base = p.ws + (static_cast<size_t>(pair) * p.max_contrib + (cta - contrib_first)) * (n_out + G);
        for (int idx = tid; idx < n_out; idx += kComputeWarps * 32) {
            const int gg = idx / D;
            const int d = idx % D;
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < kComputeWarps; ++w)
                M = fmaxf(M, red_m[w * G + gg]);
            float L = 0.f, O = 0.f;
#pragma unroll
            for (int w = 0; w < kComputeWarps; ++w) {
                const float mw = red_m[w * G + gg];
                const float e = (mw == -INFINITY) ? 0.f : ex2(mw - M);
                L = fmaf(red_l[w * G + gg], e, L);
                O = fmaf(red_o[(w * G + gg) * D + d], e, O);
            }
            const size_t bh = static_cast<size_t>(b) * p.Hq + h0 + gg;
            if (whole_pair) {
                p.o[bh * D + d] = __float2bfloat16_rn(O / L);
                if (d == 0)
                    p.lse[bh] = (M + log2f(L)) * kLn2;
            } else {
                slot_base[idx] = O / L;
                if (d == 0)
                    slot_base[n_out + gg] = M + log2f(L);
            }
        }

        if (!whole_pair && tid == 0) {
            // Signalled once the whole range is streamed (see below): only the first and the last
            // segment of a range can be a piece of a shared pair.
            deferred_pair[n_deferred] = pair;
            deferred_first[n_deferred] = contrib_first;
            ++n_deferred;
        }
        named_sync_compute<kComputeWarps * 32>();  // shared merge buffers and the flag are reused by the next segment
        g = seg_end;
    }

    // ---------------------------------------------------------------- shared pairs: the last CTA merges
    // Every partial this CTA wrote is published by one fence, then each shared pair's arrival counter
    // is bumped; the CTA that brings a counter to the pair's contributor count merges its partials.
    int n_def = 0;
    if (tid == 0) {
        n_def = n_deferred;
        if (n_def > 0)
            __threadfence();
        for (int k = 0; k < n_def; ++k) {
            const long long pr = deferred_pair[k];
            const int first = deferred_first[k];
            const int n_contrib = cta_of_unit((pr + 1) * p.cpp - 1, p.total, p.ctas) - first + 1;
            const int prev = atomicAdd(&p.counters[pr], 1);
            last_flag[k] = (prev == n_contrib - 1) ? n_contrib : 0;
        }
        last_flag[2] = n_def;
    }
    named_sync_compute<kComputeWarps * 32>();
    n_def = last_flag[2];
    for (int k = 0; k < n_def; ++k) {
        const int n_contrib = last_flag[k];
        if (n_contrib == 0)
            continue;
        __threadfence();
        const long long pr = deferred_pair[k];
        const long long bk = pr / p.head_groups;
        const long long b = bk / p.Hkv;
        const int h0 = static_cast<int>(bk % p.Hkv) * p.group + static_cast<int>(pr % p.head_groups) * G;
        const float *pbase = p.ws + static_cast<size_t>(pr) * p.max_contrib * (n_out + G);
        for (int idx = tid; idx < n_out; idx += kComputeWarps * 32) {
            const int gg = idx / D;
            const int d = idx % D;
            float M = -INFINITY;
            for (int s = 0; s < n_contrib; ++s)
                M = fmaxf(M, __ldcg(pbase + s * (n_out + G) + n_out + gg));
            float W = 0.f, O = 0.f;
            for (int s = 0; s < n_contrib; ++s) {
                const float w = ex2(__ldcg(pbase + s * (n_out + G) + n_out + gg) - M);
                W += w;
                O = fmaf(w, __ldcg(pbase + s * (n_out + G) + idx), O);
            }
            const size_t bh = static_cast<size_t>(b) * p.Hq + h0 + gg;
            p.o[bh * D + d] = __float2bfloat16_rn(O / W);
            if (d == 0)
                p.lse[bh] = (M + log2f(W)) * kLn2;
        }
        if (tid == 0)
            atomicExch(&p.counters[pr], 0);  // ready for the next call
    }
}

template <int D, int G>
cudaError_t prepare_dg(int *ctas_per_sm)
{
    using C = DecCfg<D, G>;
    static int cached_per_dev[kMaxDevices] = {};  // per device: attributes apply to the current one
    const int dev = current_device_index();
    if (dev < 0)
        return cudaErrorInvalidDevice;
    int &cached = cached_per_dev[dev];
    if (cached == 0) {
        cudaError_t e = cudaFuncSetAttribute(decode_kernel<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(decode_kernel<D, G>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                     cudaSharedmemCarveoutMaxShared);
        int n = 0;
        if (e == cudaSuccess)
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_kernel<D, G>, C::kThreads, C::kSmem);
        if (e != cudaSuccess)
            return e;
        cached = n > 0 ? n : 1;
    }
    if (ctas_per_sm)
        *ctas_per_sm = cached;
    return cudaSuccess;
}

template <int D, int G>
cudaError_t launch_dg(const DecodeArgs &a, cudaStream_t stream)
{
    using C = DecCfg<D, G>;
    cudaError_t e = prepare_dg<D, G>(nullptr);
    if (e != cudaSuccess)
        return e;
    const DecodePlan &pl = a.plan;
    Params p;
    p.q = static_cast<const __nv_bfloat16 *>(a.q);
    p.k = static_cast<const __nv_bfloat16 *>(a.k);
    p.v = static_cast<const __nv_bfloat16 *>(a.v);
    p.o = static_cast<__nv_bfloat16 *>(a.o);
    p.lse = a.lse;
    p.ws = a.ws;
    p.counters = a.counters;
    p.status = a.status;
    p.Hq = a.Hq;
    p.Hkv = a.Hkv;
    p.Skv = a.Skv;
    p.group = a.Hq / a.Hkv;
    p.head_groups = pl.head_groups;
    p.cpp = pl.cpp;
    p.ctas = pl.ctas;
    p.max_contrib = pl.max_contrib;
    p.total = pl.total;
    p.scale_log2 = a.scale * kLog2e;
    decode_kernel<D, G><<<static_cast<unsigned>(pl.ctas), C::kThreads, C::kSmem, stream>>>(p);
    return cudaGetLastError();
}

template <int D>
cudaError_t dispatch_d(int G, const DecodeArgs *a, cudaStream_t stream, int *ctas_per_sm)
{
    switch (G) {
    case 1:
        return a ? launch_dg<D, 1>(*a, stream) : prepare_dg<D, 1>(ctas_per_sm);
    case 2:
        return a ? launch_dg<D, 2>(*a, stream) : prepare_dg<D, 2>(ctas_per_sm);
    case 4:
        return a ? launch_dg<D, 4>(*a, stream) : prepare_dg<D, 4>(ctas_per_sm);
    default:
        return a ? launch_dg<D, 8>(*a, stream) : prepare_dg<D, 8>(ctas_per_sm);
    }
}

cudaError_t dispatch(int D, int G, const DecodeArgs *a, cudaStream_t stream, int *ctas_per_sm)
{
    switch (D) {
    case 32:
        return dispatch_d<32>(G, a, stream, ctas_per_sm);
    case 64:
        return dispatch_d<64>(G, a, stream, ctas_per_sm);
    case 128:
        if (a)
            return launch_decode_tc(*a, stream);
        return decode_tc_ctas_per_sm(G, false, ctas_per_sm);
    default:
        return cudaErrorInvalidValue;
    }
}

}  // namespace

int decode_heads_per_cta(int group, int D)
{
    if (D == 128)
        return decode_tc_heads_per_pair(group);
    // Largest power of two that divides the group size, at most 8.
    const int cap = 8;
    int g = 1;
    while (g < cap && group % (2 * g) == 0)
        g *= 2;
    return g;
}

cudaError_t decode_plan(int B, int Hq, int Hkv, int Skv, int D, int requested_ctas, int sm_count, DecodePlan *plan,
                        bool fp8)
{
    DecodePlan pl;
    const int group = Hq / Hkv;
    pl.G = decode_heads_per_cta(group, D);
    pl.head_groups = group / pl.G;
    pl.pairs = static_cast<long long>(B) * Hkv * pl.head_groups;
    pl.ck = (D == 128) ? decode_tc_chunk_keys() : keys_per_stage(pl.G);
    pl.cpp = (Skv + pl.ck - 1) / pl.ck;
    pl.total = pl.pairs * pl.cpp;
    long long ctas = requested_ctas;
    if (ctas <= 0) {
        int per_sm = 1;
        const cudaError_t e = (D == 128) ? decode_tc_ctas_per_sm(pl.G, fp8, &per_sm)
                                         : dispatch(D, pl.G, nullptr, nullptr, &per_sm);
        if (e != cudaSuccess)
            return e;
        const long long slots = static_cast<long long>(sm_count) * per_sm;
        // One CTA per resident slot, except when whole pairs already fill most of the slots:
        // sharing a pair costs a merge, which measured dearer than leaving a few SMs idle.
        ctas = (pl.pairs <= slots && 4 * pl.pairs >= 3 * slots) ? pl.pairs : slots;
    }
    if (ctas > pl.total)
        ctas = pl.total;
    // range_start multiplies a CTA index by the unit count: keep the product inside 63 bits.
    if (ctas > (1LL << 22) || pl.total > (1LL << 40))
        return cudaErrorInvalidValue;
    pl.ctas = static_cast<int>(ctas);
    const long long per = pl.total / pl.ctas;  // >= 1 unit per CTA
    // Pairs are shared between CTAs unless every range is a whole number of pairs.
    const bool shared = !(pl.total % pl.ctas == 0 && per % pl.cpp == 0);
    long long mc = (pl.cpp + per - 1) / per + 1;
    if (mc > pl.ctas)
        mc = pl.ctas;
    pl.max_contrib = shared ? static_cast<int>(mc) : 1;
    if (D == 128)  // the tensor-core kernel keeps at most two partials per CTA
        pl.partial_floats = shared ? decode_tc_partial_floats(pl.G, pl.ctas) : 0;
    else
        pl.partial_floats =
            shared ? static_cast<size_t>(pl.pairs) * pl.max_contrib * (static_cast<size_t>(pl.G) * D + pl.G) : 0;
    *plan = pl;
    return cudaSuccess;
}

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream)
{
    return dispatch(a.D, a.plan.G, &a, stream, nullptr);
}

}  // namespace attn_b200
