/*
 * decode_tc_sm100.cu — attention of one new query token per (batch, query head) over a bf16 K/V
 * cache (Sq == 1) with head dim 128, on the tensor core.
 *
 * Work split: as the CUDA-core decode kernel (decode_sm100.cu). A "pair" is one (batch, kv head,
 * group of G query heads sharing that kv head), its keys are cut into chunks of 128, all pairs'
 * chunks are laid end to end and CTA c of the launched CTAs streams the units
 * [c*T/P, (c+1)*T/P); a CTA that holds a whole pair writes its output, the pieces of a shared pair
 * are merged by whichever contributing CTA finishes last: M = max_s LSE_s,
 * LSE = M + log2 sum_s 2^(LSE_s - M), O = sum_s 2^(LSE_s - LSE) O_s.
 *
 * Per chunk of 128 keys (K_c, V_c: 128 x 128 bf16 each, TMA-loaded with 128-byte swizzle):
 *
 *   S^T = K_c Q^T     tcgen05.mma, M = 128 keys, N = 16 (the G query heads, padded), K = 128 dims;
 *                     fp32 scores in tensor memory, key i in TMEM lane i;
 *   softmax           thread i owns key i: it scales its G scores to log2 units; the chunk's max
 *                     per head comes from a warp butterfly and one exchange between the four
 *                     warps; the reference max m moves only when a head's max exceeds it by more
 *                     than 8 (then the O accumulator and the running sums are scaled by
 *                     2^(m_old - m_new)); the weights 2^(s - m), rounded to bf16, go to shared
 *                     memory as P^T (16 x 128, K-major, 128-byte swizzle);
 *   O^T += V_c^T P^T  tcgen05.mma, M = 128 dims (A = V_c read MN-major), N = 16 heads, K = 128 keys.
 *
 * The softmax works in rounds of kRound chunks (one; the loop is written for more): a round's S^T
 * are committed together and its PV products issued together. After the first round of a segment
 * the warps exchange their maxima only when some key passes the rescale threshold (a counting
 * barrier decides).
 *
 * The tensor core takes the dot products, so each key costs the CUDA cores a handful of
 * instructions per head and the kernel streams K/V at memory speed. S^T is double-buffered in
 * TMEM and P^T in shared memory: S^T of chunk c+1 is computed while the softmax of chunk c runs.
 * Each thread keeps two running sums per head over the keys it owned: of the fp32 weights (gives
 * the LSE) and of the bf16-rounded weights the PV product used (normalises O).
 *
 * Warp roles (192 threads, one CTA per SM): warps 0-3 softmax and epilogue (thread i = TMEM lane
 * i), warp 4 TMA producer, warp 5 TMEM allocator and MMA issuer (whole warp walks the schedule,
 * one elected lane issues).
 *
 * Sources (page title, section): decode attends to every cached key, no mask needed — "AI Infra
 * 入门：RMSNorm、Softmax、Causal Mask、Sampling 的数学与底层优化", §3; Flash-Decoding split-K merged by
 * LSE — same page, §3 (LSE paragraph); grouped query heads sharing a K/V head and decode being
 * bound by reading K/V — "05 · Tích vô hướng, Softmax và toán của Attention", §4; running max and
 * sum with rescale — same page §6 and "Bộ 06 · Bên trong model", Q1.
 */
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <cmath>

#include "kernels.h"
#include "sm100_ptx.cuh"
#include "tma_host.h"

namespace attn_b200 {
namespace {

constexpr int kD = 128;         // head dim (the only one this kernel serves)
constexpr int kCK = 128;        // keys per chunk = M of S^T = K of O^T
constexpr int kN = 16;          // MMA N: query heads of one pair, padded
constexpr int kWarpTma = 4;
constexpr int kWarpMma = 5;
constexpr int kSoftmaxThreads = 128;
constexpr int kThreads = 192;
constexpr int kBarSoftmax = 1;  // named barrier of the softmax warps
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

constexpr int kHalfBytes = kCK * 128;  // 128 rows x 128 bytes: one swizzled box column of a K or V chunk
constexpr int kSmallHalf = kN * 128;   // 16 rows x 128 bytes: half of a bf16 Q^T or P^T, or one e4m3 part
constexpr int kMaxStages = 5;
enum TcBar : int {
    kBarFull0 = 0,                         // [stage] K/V chunk landed
    kBarEmpty0 = kBarFull0 + kMaxStages,   // [stage] chunk consumed by both MMAs
    kBarQFull0 = kBarEmpty0 + kMaxStages,  // [segment parity] Q^T in place
    kBarQEmpty0 = kBarQFull0 + 2,          // [segment parity] last S^T of the segment done
    kBarSFull0 = kBarQEmpty0 + 2,          // [chunk parity] S^T ready
    kBarPFull0 = kBarSFull0 + 2,           // [chunk parity] P^T written (128 arrivals)
    kBarODone0 = kBarPFull0 + 2,           // [chunk parity] O^T += V^T P^T done
    kBarOFree = kBarODone0 + 2,            // segment's O^T read out (128 arrivals)
    kBarDrain = kBarOFree + 1,
    kBarQScFree0 = kBarDrain + 1,          // [segment parity] e4m3 cache: the score scales read (128 arrivals)
    kNumTcBars = kBarQScFree0 + 2,
};

// Shared-memory layout of one variant. bf16 cache: K and V chunks of 32 KB (two 64-dim box
// columns each), three in flight, Q^T and P^T in bf16. e4m3 cache: chunks of 16 KB (one 128-byte
// box column), five in flight, Q^T and P^T each as three e4m3 parts (hi, mid, lo) of 16 x 128 bytes.
// One CTA per SM either way (two smaller CTAs per SM measured slower for the e4m3 cache: pairs then
// have to be split between CTAs and merged).
template <bool kFp8>
struct Lay {
    static constexpr int kStages = kFp8 ? 5 : 3;
    static constexpr int kBoxCols = kFp8 ? 1 : 2;          // 128-byte box columns per K or V row
    static constexpr int kTileBytes = kBoxCols * kHalfBytes;  // one K or V chunk
    static constexpr int kStageBytes = 2 * kTileBytes;        // K chunk, then V chunk
    static constexpr int kSmallBytes = kFp8 ? 3 * kSmallHalf : 2 * kSmallHalf;  // one Q^T slot, one chunk's P^T
    // Chunks per softmax round (the S^T of a round's chunks is committed together and their PV
    // products issued together). One for both caches: two-chunk rounds measured slower for the e4m3
    // cache (41.0 -> 45.1 us), the issuer then holding four of the five ring stages.
    static constexpr int kRound = 1;
    static constexpr int kOffRing = 0;
    static constexpr int kOffQ = kOffRing + kStages * kStageBytes;  // two Q^T slots (one per segment parity)
    static constexpr int kOffP = kOffQ + 2 * kSmallBytes;           // two P^T buffers (one per round parity)
    static constexpr int kOffQScale = kOffP + 2 * kRound * kSmallBytes;  // [segment parity][head] score scales
    static constexpr int kOffRedMax = kOffQScale + 2 * kN * 4;      // [chunk parity][warp][head] chunk maxima
    static constexpr int kOffRedSum = kOffRedMax + 2 * 4 * kN * 4;  // [warp][head][2] running sums
    static constexpr int kOffBar = kOffRedSum + 4 * kN * 2 * 4;
    static constexpr int kOffMisc = kOffBar + kNumTcBars * 8;  // tmem slot, abort flag, merge bookkeeping
    // Paged decode only: first unit of each batch entry (and the total), then the clamped lengths.
    static constexpr int kOffBatchStart = kOffMisc + 64;
    static constexpr int kOffBatchLen = kOffBatchStart + 8 * (kPagedMaxBatch + 1);
    static constexpr int kUsed = kOffBatchLen + 4 * kPagedMaxBatch;
    static constexpr int kSmem = kUsed + 1024;  // + alignment of the base to the 1024-byte swizzle repeat
    static_assert(kSmem <= 227 * 1024, "shared memory budget");
    static_assert(kOffQ % 1024 == 0 && kOffP % 1024 == 0 && kSmallBytes % 1024 == 0,
                  "swizzled tiles sit on 1024-byte boundaries");
    static_assert(kStages <= kMaxStages, "barrier arrays");
    // The MMA issuer holds a round's chunks until the next round's S^T is issued: two rounds in the ring.
    static_assert(kStages >= 2 * kRound, "ring deep enough for two rounds");
    // The reference max moves when a chunk's max exceeds it by more than this (log2 units). With the
    // e4m3 cache the weights are scaled by 16 before they are split, and 16 * 2^4 = 256 stays below
    // the e4m3 maximum of 448.
    static constexpr float kRescaleThreshold = kFp8 ? 4.0f : 8.0f;
    static constexpr float kPScale = kFp8 ? 16.0f : 1.0f;
};
static_assert(Lay<false>::kStageBytes == 65536 && Lay<false>::kSmallBytes == 4096, "bf16 layout");
// TMEM: S^T of a round's chunks [round parity][slot] in 16-column groups from column 0, then O^T.
// With the e4m3 cache every product is a sum over three e4m3 parts (of Q^T or of P^T); each part
// accumulates in its own 16 columns (one N = 48 instruction per K step computes all three), and
// the readers add the parts.
template <bool kFp8>
struct TmemLay {
    static constexpr int kRound = Lay<kFp8>::kRound;
    static constexpr int kParts = kFp8 ? 3 : 1;
    static constexpr uint32_t kColO = 32u * kRound * kParts;       // after the double-buffered S^T of the rounds
    static constexpr uint32_t kCols = (kColO + 16u * kParts <= 64u) ? 64u : (kColO + 16u * kParts <= 128u) ? 128u : 256u;
    __host__ __device__ static constexpr uint32_t col_s(int parity, int slot)
    {
        return 16u * static_cast<uint32_t>((kRound * parity + slot) * kParts);
    }
};

struct TcParams {
    __nv_bfloat16 *o;
    long long o_sb, o_sh;  // element strides of o (batch, head); each head's D values are contiguous
    long long q_sb, q_sh;  // element strides of q (batch, head), read directly by the e4m3 producer
    float *lse;
    float *ws;  // partials: [CTA][first or last segment][G*D + G]
    int *counters, *status;
    int Hq, Hkv, Skv, group, head_groups, cpp, ctas;
    long long total;
    float scale_log2;
    // paged, variable-length cache
    const int *seq_lens, *block_table;
    int B, num_pages, page_size, pages_per_seq, max_seq_len;
    // e4m3 cache: the bf16 queries, read by the producer, and the per-(kv head, channel) coefficients
    const __nv_bfloat16 *q;
    const float *k_scale, *v_scale;
};

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ---- e4m3 cache: splitting a fp32 value into three e4m3 parts ---------------------------------
// x ~ c1 + c2 + c3 with c_t = e4m3(x - c1 - ... - c_{t-1}) rounded to nearest even. Each
// subtraction is exact (a value and its 3-bit rounding lie within a factor of two of each other),
// so the parts carry x to about 12 significant bits wherever x, scaled as below, is above the
// e4m3 subnormal range (2^-6).

// Codes of (a, b), a in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float a, float b)
{
    return __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
}

__device__ __forceinline__ float2 e4m3x2_value(uint32_t codes)
{
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(codes), __NV_E4M3);
    return __half22float2(__half2(h));
}

// One split step over four values: their codes (value u in byte u), and x -= the codes' values.
__device__ __forceinline__ uint32_t split_step4(float (&x)[4])
{
    const uint32_t lo = e4m3x2(x[0], x[1]), hi = e4m3x2(x[2], x[3]);
    const float2 vl = e4m3x2_value(lo), vh = e4m3x2_value(hi);
    x[0] -= vl.x;
    x[1] -= vl.y;
    x[2] -= vh.x;
    x[3] -= vh.y;
    return lo | (hi << 16);
}

// 2^e for |e| <= 126.
__device__ __forceinline__ float exp2_int(int e) { return __uint_as_float(static_cast<uint32_t>(e + 127) << 23); }

// The power of two e that brings mx (the largest magnitude of one query head's q * k_scale) into
// (224, 448], the top of the e4m3 range: 0 for a zero head, clamped to [-100, 100].
__device__ __forceinline__ int q_exponent(float mx)
{
    if (!(mx > 0.f))
        return 0;
    const uint32_t bits = __float_as_uint(mx);
    const int E = static_cast<int>((bits >> 23) & 255u) - 127;
    const float mant = __uint_as_float((bits & 0x007fffffu) | 0x3f800000u);  // in [1, 2)
    const int e = (mant <= 1.75f ? 8 : 7) - E;
    return min(max(e, -100), 100);
}

__device__ __forceinline__ long long range_start(long long c, long long total, int ctas) { return c * total / ctas; }

// The CTA whose range holds unit g (0 <= g < total): the largest c with range_start(c) <= g.
// floor(c T / P) <= g  <=>  c < (g + 1) P / T, so c = ceil((g + 1) P / T) - 1. Exact also when
// there are fewer units than CTAs and several CTAs have empty ranges starting at the same unit.
__device__ __forceinline__ int cta_of_unit(long long g, long long total, int ctas)
{
    return static_cast<int>(((g + 1) * ctas - 1) / total);
}

// Wait that ignores the abort flag (drains copies in flight before the CTA exits).
__device__ __forceinline__ bool wait_drain(uint32_t bar, uint32_t parity, uint64_t limit_ns)
{
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > limit_ns)
            return false;
    }
    return true;
}

// Where unit g of the whole sequence of chunks falls: its pair, the chunk within the pair, the
// pair's chunk count and the pair's first unit.
struct UnitPos {
    long long pair, pair_start;
    int local, cpp;
};

template <int G, bool kPaged, bool kFp8>
__global__ void __launch_bounds__(kThreads, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const TcParams p)
{
    static_assert(G >= 1 && G <= kN, "one pair's heads fit the MMA's N");
    using L = Lay<kFp8>;
    using TL = TmemLay<kFp8>;
    constexpr int kRound = L::kRound;
    constexpr uint32_t kColO = TL::kColO;
    static_assert(TL::kRound == L::kRound, "one round size");
    constexpr int kStages = L::kStages, kStageBytes = L::kStageBytes, kTileBytes = L::kTileBytes;
    constexpr int kSmallBytes = L::kSmallBytes, kOffRing = L::kOffRing, kOffQ = L::kOffQ, kOffP = L::kOffP;
    constexpr int kOffRedMax = L::kOffRedMax, kOffRedSum = L::kOffRedSum, kOffBar = L::kOffBar;
    constexpr int kOffMisc = L::kOffMisc, kOffBatchStart = L::kOffBatchStart, kOffBatchLen = L::kOffBatchLen;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t s_base = smem_u32(smem);
    const uint32_t sRing = s_base + kOffRing;
    const uint32_t sQ = s_base + kOffQ;
    const uint32_t sP = s_base + kOffP;
    const uint32_t bar0 = s_base + kOffBar;
#define BAR(i) (bar0 + 8u * static_cast<uint32_t>(i))
    float *red_max = reinterpret_cast<float *>(smem + kOffRedMax);
    float *q_scale = reinterpret_cast<float *>(smem + L::kOffQScale);  // [segment parity][kN], e4m3 cache
    float *red_sum = reinterpret_cast<float *>(smem + kOffRedSum);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffMisc + 4);
    int *last_flag = reinterpret_cast<int *>(smem + kOffMisc + 8);                     // [3]
    long long *deferred_pair = reinterpret_cast<long long *>(smem + kOffMisc + 24);    // [2]
    int *deferred_first = reinterpret_cast<int *>(smem + kOffMisc + 40);              // [2]

    long long *batch_start = reinterpret_cast<long long *>(smem + kOffBatchStart);  // [B + 1]
    int *batch_len = reinterpret_cast<int *>(smem + kOffBatchLen);                   // [B]

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int cta = blockIdx.x;
    const int pairs_per_b = p.Hkv * p.head_groups;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(BAR(kBarFull0 + s), 1);
            mbar_init(BAR(kBarEmpty0 + s), 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(BAR(kBarQFull0 + x), kFp8 ? 32 : 1);  // e4m3: every producer lane writes Q^T
            mbar_init(BAR(kBarQScFree0 + x), kSoftmaxThreads);
            mbar_init(BAR(kBarQEmpty0 + x), 1);
            mbar_init(BAR(kBarSFull0 + x), 1);
            mbar_init(BAR(kBarPFull0 + x), kSoftmaxThreads);
            mbar_init(BAR(kBarODone0 + x), 1);
        }
        mbar_init(BAR(kBarOFree), kSoftmaxThreads);
        mbar_init(BAR(kBarDrain), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    // P^T rows G..15 are never written by the softmax, nor (e4m3 cache) Q^T rows G..15 by the
    // producer: keep them zero. Q^T and P^T are adjacent.
    {
        constexpr int kZeroFrom = kFp8 ? kOffQ : kOffP;
        for (int i = threadIdx.x; i < (kOffP + 2 * L::kRound * kSmallBytes - kZeroFrom) / 16; i += kThreads)
            reinterpret_cast<uint4 *>(smem + kZeroFrom)[i] = make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
    if (warp == kWarpTma && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    if (warp == kWarpMma) {
        tmem_alloc(smem_u32(tmem_slot), TmemLay<kFp8>::kCols);
        tmem_relinquish();
    }
    if constexpr (kPaged) {
        // Each batch entry's length, clamped to what its block-table row and the workspace (sized
        // for max_seq_len) can hold, and the first unit of its chunks (an exclusive scan by warp 0).
        const int cap = min(p.max_seq_len, p.pages_per_seq * p.page_size);
        for (int b = threadIdx.x; b < p.B; b += kThreads)
            batch_len[b] = min(max(p.seq_lens[b], 0), cap);
        __syncthreads();
        if (warp == 0) {
            long long running = 0;
            for (int base = 0; base < p.B; base += 32) {
                const int b = base + lane;
                const long long u = (b < p.B) ? static_cast<long long>(pairs_per_b) * ((batch_len[b] + kCK - 1) / kCK) : 0;
                long long incl = u;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const long long y = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o)
                        incl += y;
                }
                if (b < p.B)
                    batch_start[b] = running + incl - u;
                running += __shfl_sync(0xffffffffu, incl, 31);
            }
            if (lane == 0)
                batch_start[p.B] = running;
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const long long total = kPaged ? batch_start[p.B] : p.total;
    const long long g_begin = range_start(cta, total, p.ctas);
    const long long g_end = range_start(cta + 1, total, p.ctas);

    auto locate = [&](long long g) -> UnitPos {
        UnitPos u;
        if constexpr (kPaged) {
            // The batch entry holding unit g: the largest b with batch_start[b] <= g (an entry with
            // no chunks never qualifies, because the next entry starts at the same unit).
            int lo = 0, hi = p.B - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (batch_start[mid] <= g)
                    lo = mid;
                else
                    hi = mid - 1;
            }
            u.cpp = (batch_len[lo] + kCK - 1) / kCK;
            const long long w = g - batch_start[lo];
            const long long in_b = w / u.cpp;
            u.pair = static_cast<long long>(lo) * pairs_per_b + in_b;
            u.local = static_cast<int>(w - in_b * u.cpp);
            u.pair_start = batch_start[lo] + in_b * u.cpp;
        } else {
            u.cpp = p.cpp;
            u.pair = g / p.cpp;
            u.local = static_cast<int>(g - u.pair * p.cpp);
            u.pair_start = u.pair * p.cpp;
        }
        return u;
    };
    auto pair_first_unit = [&](long long pair, int *cpp) -> long long {
        if constexpr (kPaged) {
            const int b = static_cast<int>(pair / pairs_per_b);
            *cpp = (batch_len[b] + kCK - 1) / kCK;
            return batch_start[b] + (pair - static_cast<long long>(b) * pairs_per_b) * *cpp;
        } else {
            *cpp = p.cpp;
            return pair * p.cpp;
        }
    };

    if (warp == kWarpTma) {
        // ---------------------------------------------------------------- TMA producer
        // The whole warp walks the schedule (waits agreed with __all_sync); lane 0 issues the
        // copies. For a paged cache each lane keeps one block-table entry of a 32-entry window, so
        // the table costs one coalesced load per 32 pages instead of a dependent load per page.
        const bool issuer = (lane == 0);
        int issued = 0, seg = 0;
        UnitPos pos = locate(g_begin);
        long long pair = pos.pair;
        int local = pos.local, cpp = pos.cpp;
        int bk = 0;
        int tab_row = -1, tab_base = 0, tab_val = 0;  // this lane holds entry tab_base + lane of row tab_row
        for (long long g = g_begin; g < g_end; ++g) {
            const bool new_seg = (g == g_begin || local == 0);
            const int qs = seg & 1;
            uint2 qraw[kFp8 ? G : 1];  // e4m3 cache: this lane's dims 4*lane .. 4*lane+3 of each head
            float4 ksv = make_float4(0.f, 0.f, 0.f, 0.f);
            if (new_seg) {
                // A new segment: Q^T of its pair (G heads, padded to 16 rows) into the segment's slot.
                const uint32_t free_parity = (static_cast<uint32_t>(seg >> 1) & 1u) ^ 1u;
                if (!__all_sync(0xffffffffu, mbar_wait(BAR(kBarQEmpty0 + qs), free_parity, abort_flag, p.status,
                                                       kSiteDecodeProducer)))
                    break;
                // e4m3 cache: the softmax warps also have read the slot's score scales.
                if (kFp8 && !__all_sync(0xffffffffu, mbar_wait(BAR(kBarQScFree0 + qs), free_parity, abort_flag,
                                                               p.status, kSiteDecodeProducer)))
                    break;
                const int hg = static_cast<int>(pair % p.head_groups);
                bk = static_cast<int>(pair / p.head_groups);  // b * Hkv + kv head
                const int b = bk / p.Hkv;
                const int h0 = (bk % p.Hkv) * p.group + hg * G;
                if constexpr (kFp8) {
                    // Loads only; Q^T is built once this chunk's copies are on their way.
                    const __nv_bfloat16 *qrow = p.q + b * p.q_sb + h0 * p.q_sh;
#pragma unroll
                    for (int h = 0; h < (kFp8 ? G : 1); ++h)
                        qraw[h] = reinterpret_cast<const uint2 *>(qrow + h * p.q_sh)[lane];
                    ksv = reinterpret_cast<const float4 *>(p.k_scale + static_cast<size_t>(bk % p.Hkv) * kD)[lane];
                } else if (issuer) {
                    mbar_arrive_expect_tx(BAR(kBarQFull0 + qs), kSmallBytes);
                    for (int hf = 0; hf < 2; ++hf)
                        tma_load_4d(sQ + qs * kSmallBytes + hf * kSmallHalf, &tm_q, BAR(kBarQFull0 + qs), hf * 64,
                                    h0, 0, b);
                }
                ++seg;
            }
            const int slot = issued % kStages;
            if (!__all_sync(0xffffffffu, mbar_wait(BAR(kBarEmpty0 + slot), (static_cast<uint32_t>(issued / kStages) & 1u) ^ 1u,
                                                   abort_flag, p.status, kSiteDecodeProducer)))
                break;
            const uint32_t dst = sRing + slot * kStageBytes;
            const int key0 = local * kCK;
            if (issuer)
                mbar_arrive_expect_tx(BAR(kBarFull0 + slot), kStageBytes);
            if constexpr (kPaged) {
                // The chunk's keys come page by page: boxes of min(page_size, 128) rows, box l issued
                // by lane l so that small pages do not queue behind one thread. A box past the
                // sequence's length reads the page beyond the last one, which the map fills with
                // zeros, and never touches the block table past its row.
                const int b = bk / p.Hkv;
                const int kvh = bk - b * p.Hkv;
                const int rows = min(p.page_size, kCK);
                const int n_box = kCK / rows;
                const int e0 = key0 / p.page_size;  // block-table entry of the chunk's first key
                if (b != tab_row || e0 < tab_base || e0 + n_box > tab_base + 32) {  // the same in every lane
                    tab_row = b;
                    tab_base = e0;
                    const int idx = e0 + lane;
                    tab_val = (idx < p.pages_per_seq) ? p.block_table[static_cast<size_t>(b) * p.pages_per_seq + idx]
                                                      : p.num_pages;
                }
                const int key = key0 + lane * rows;
                const int e = (lane < n_box) ? key / p.page_size : e0;
                int page = __shfl_sync(0xffffffffu, tab_val, e - tab_base);
                if (lane < n_box) {
                    // Keys past the length, and a table entry outside [0, num_pages) (which could
                    // otherwise wrap page * Hkv onto another sequence's page), read the zero-filled
                    // page beyond the last one.
                    if (key >= batch_len[b] || page < 0 || page >= p.num_pages)
                        page = p.num_pages;
                    const int in_page = key % p.page_size;
                    for (int hf = 0; hf < L::kBoxCols; ++hf) {
                        tma_load_4d(dst + hf * kHalfBytes + lane * rows * 128, &tm_k, BAR(kBarFull0 + slot), hf * 64,
                                    in_page, kvh, page);
                        tma_load_4d(dst + kTileBytes + hf * kHalfBytes + lane * rows * 128, &tm_v, BAR(kBarFull0 + slot),
                                    hf * 64, in_page, kvh, page);
                    }
                }
            } else if (issuer) {
                for (int hf = 0; hf < L::kBoxCols; ++hf) {
                    tma_load_4d(dst + hf * kHalfBytes, &tm_k, BAR(kBarFull0 + slot), hf * 64, key0, bk % p.Hkv,
                                bk / p.Hkv);
                    tma_load_4d(dst + kTileBytes + hf * kHalfBytes, &tm_v, BAR(kBarFull0 + slot), hf * 64, key0,
                                bk % p.Hkv, bk / p.Hkv);
                }
            }
            if constexpr (kFp8) {
                if (new_seg) {
                    // Q^T parts: per head, q * k_scale scaled by 2^e into the top of the e4m3 range,
                    // then split into three e4m3 parts (rows h of three 16 x 128-byte K-major tiles
                    // with the 128-byte swizzle: dims 4*lane..4*lane+3 sit in 16-byte unit
                    // (lane / 4) XOR (h % 8), bytes 4*(lane % 4)..+3). The scores come out scaled by
                    // 2^e; the softmax undoes that with the factor left in q_scale.
                    uint8_t *qbase = smem + kOffQ + qs * kSmallBytes;
                    const uint32_t unit = static_cast<uint32_t>(lane >> 2), sub = static_cast<uint32_t>(lane & 3) * 4u;
                    auto lo = [](uint32_t w) { return __uint_as_float(w << 16); };
                    auto hi = [](uint32_t w) { return __uint_as_float(w & 0xffff0000u); };
#pragma unroll
                    for (int h = 0; h < (kFp8 ? G : 1); ++h) {
                        float x[4] = {lo(qraw[h].x) * ksv.x, hi(qraw[h].x) * ksv.y, lo(qraw[h].y) * ksv.z,
                                      hi(qraw[h].y) * ksv.w};
                        float mx = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1)
                            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                        const int e = q_exponent(mx);
                        const float f = exp2_int(e);
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            x[u] *= f;
                        const uint32_t off = static_cast<uint32_t>((h >> 3) * 1024 + (h & 7) * 128) +
                                             (((unit ^ static_cast<uint32_t>(h & 7)) << 4) | sub);
#pragma unroll
                        for (int t = 0; t < 3; ++t)
                            *reinterpret_cast<uint32_t *>(qbase + t * kSmallHalf + off) = split_step4(x);
                        if (lane == 0)
                            q_scale[qs * kN + h] = p.scale_log2 * exp2_int(-e);
                    }
                    fence_proxy_async_smem();
                    mbar_arrive(BAR(kBarQFull0 + qs));
                }
            }
            ++issued;
            if (++local == cpp && g + 1 < g_end) {
                pos = locate(g + 1);
                pair = pos.pair;
                local = pos.local;
                cpp = pos.cpp;
            }
        }
        if (*abort_flag && issuer) {
            // Let every copy already issued land before the CTA exits.
            for (int c = (issued > kStages ? issued - kStages : 0); c < issued; ++c)
                wait_drain(BAR(kBarFull0 + c % kStages), static_cast<uint32_t>(c / kStages) & 1u, 100000000ull);
            for (int s = (seg > 2 ? seg - 2 : 0); !kFp8 && s < seg; ++s)  // e4m3 Q^T is not copied by TMA
                wait_drain(BAR(kBarQFull0 + (s & 1)), static_cast<uint32_t>(s >> 1) & 1u, 100000000ull);
        }
    } else if (warp == kWarpMma) {
        // ---------------------------------------------------------------- MMA issuer
        // A = K chunk, B = Q^T; then A = V chunk read MN-major, B = P^T. e4m3 cache: both operands e4m3.
        // e4m3: the three parts of Q^T (or of P^T) sit one after another (16 rows each, 8-row groups
        // 1024 bytes apart), so one instruction of N = 48 takes all three, each part's product
        // landing in its own 16 accumulator columns.
        constexpr int kNP = kFp8 ? 3 * kN : kN;
        constexpr uint32_t kIdS = kFp8 ? idesc_e4m3_f32_ab(kCK, kNP, false, false) : idesc_bf16_f32_ab(kCK, kN, false, false);
        constexpr uint32_t kIdO = kFp8 ? idesc_e4m3_f32_ab(kD, kNP, true, false) : idesc_bf16_f32_ab(kD, kN, true, false);
        const bool leader = elect_one();
        // A K step moves the start address, the low field of a descriptor (address >> 4): every
        // address here is below 2^18, so the field never overflows.
        const uint64_t desc_k0 = smem_desc(sRing, 16, 1024, kSwizzle128B);
        const uint64_t desc_v0 = smem_desc(sRing + kTileBytes, kHalfBytes, 1024, kSwizzle128B);
        const uint64_t desc_q0 = smem_desc(sQ, 16, 1024, kSwizzle128B);
        const uint64_t desc_p0 = smem_desc(sP, 16, 1024, kSwizzle128B);
        auto commit = [&](int bar) {
            if (leader)
                tc_commit(BAR(bar));
        };
        // S^T of chunk c (ring stage c % kStages) against the segment's Q^T slot qs, into TMEM column dcol.
        auto issue_s = [&](int c, int qs, uint32_t dcol) {
            const uint64_t dk = desc_k0 + static_cast<uint64_t>((c % kStages) * (kStageBytes >> 4));
            const uint64_t dq = desc_q0 + static_cast<uint64_t>(qs * (kSmallBytes >> 4));
            if constexpr (kFp8) {
                // [K Q^T_hi | K Q^T_mid | K Q^T_lo]: four K steps of 32 dims (32 bytes).
                if (leader) {
#pragma unroll
                    for (int kk = 0; kk < kD / 32; ++kk)
                        tc_mma_f8_ss(tmem + dcol, dk + static_cast<uint64_t>((kk * 32) >> 4),
                                     dq + static_cast<uint64_t>((kk * 32) >> 4), kIdS, kk > 0 ? 1u : 0u);
                }
                return;
            }
            if (leader) {
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint64_t oa = static_cast<uint64_t>(((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4);
                    const uint64_t ob = static_cast<uint64_t>(((kk >> 2) * kSmallHalf + (kk & 3) * 32) >> 4);
                    tc_mma_ss(tmem + dcol, dk + oa, dq + ob, kIdS, kk > 0 ? 1u : 0u);
                }
            }
        };
        // O^T += V_c^T P^T with P^T from buffer (round parity rp, slot).
        auto issue_o = [&](int c, int rp, int slot, bool accumulate) {
            const uint64_t dv = desc_v0 + static_cast<uint64_t>((c % kStages) * (kStageBytes >> 4));
            const uint64_t dp = desc_p0 + static_cast<uint64_t>((rp * kRound + slot) * (kSmallBytes >> 4));
            if constexpr (kFp8) {
                // [O^T_hi | O^T_mid | O^T_lo] += V^T [P^T_hi | P^T_mid | P^T_lo]: four K steps of 32
                // keys (32 rows of 128 bytes of the MN-major V chunk; 32 bytes of a P^T row).
                if (leader) {
#pragma unroll
                    for (int kk = 0; kk < kCK / 32; ++kk)
                        tc_mma_f8_ss(tmem + kColO, dv + static_cast<uint64_t>((kk * 32 * 128) >> 4),
                                     dp + static_cast<uint64_t>((kk * 32) >> 4), kIdO, (accumulate || kk > 0) ? 1u : 0u);
                }
                return;
            }
            if (leader) {
#pragma unroll
                for (int kk = 0; kk < kCK / 16; ++kk) {
                    const uint64_t oa = static_cast<uint64_t>((kk * 16 * 128) >> 4);  // 16 keys of 128-byte rows
                    const uint64_t ob = static_cast<uint64_t>(((kk >> 2) * kSmallHalf + (kk & 3) * 32) >> 4);
                    tc_mma_ss(tmem + kColO, dv + oa, dp + ob, kIdO, (accumulate || kk > 0) ? 1u : 0u);
                }
            }
        };
        // The PV products of round rnd (chunks c0 .. c0 + nk - 1) once its weights are written; a
        // segment's first round overwrites O^T, after the previous segment's O^T has been read out.
        auto finish_round = [&](int rnd, int c0, int nk, bool first, int sg) -> bool {
            if (first && sg > 0 &&
                !mbar_wait(BAR(kBarOFree), static_cast<uint32_t>(sg - 1) & 1u, abort_flag, p.status, kSiteDecodeConsumer))
                return false;
            if (!mbar_wait(BAR(kBarPFull0 + (rnd & 1)), static_cast<uint32_t>(rnd >> 1) & 1u, abort_flag, p.status,
                           kSiteDecodeConsumer))
                return false;
            tc_fence_after_sync();
            for (int k = 0; k < nk; ++k)
                issue_o(c0 + k, rnd & 1, k, !first || k > 0);
            commit(kBarODone0 + (rnd & 1));
            for (int k = 0; k < nk; ++k)
                commit(kBarEmpty0 + (c0 + k) % kStages);
            return true;
        };

        // Rounds of up to kRound chunks, never across a segment boundary: all of a round's S^T are
        // committed together, then the previous round's PV products are issued.
        bool ok = true;
        int c = 0, seg = -1, rnd = -1, slot = 0, cur_c0 = 0;
        bool cur_first = false, have_prev = false, prev_first = false;
        int prev_seg = 0, prev_rnd = 0, prev_c0 = 0, prev_nk = 0;
        UnitPos pos = locate(g_begin);
        int local = pos.local, cpp = pos.cpp;
        for (long long g = g_begin; ok && g < g_end; ++g) {
            const bool first = (g == g_begin) || (local == 0);
            const bool last = (g + 1 == g_end) || (local + 1 == cpp);
            if (first) {
                ++seg;
                slot = 0;
                if (!(ok = mbar_wait(BAR(kBarQFull0 + (seg & 1)), static_cast<uint32_t>(seg >> 1) & 1u, abort_flag,
                                     p.status, kSiteDecodeConsumer)))
                    break;
            }
            if (slot == 0) {
                ++rnd;
                cur_c0 = c;
                cur_first = first;
            }
            if (!(ok = mbar_wait(BAR(kBarFull0 + c % kStages), static_cast<uint32_t>(c / kStages) & 1u, abort_flag,
                                 p.status, kSiteDecodeConsumer)))
                break;
            tc_fence_after_sync();
            issue_s(c, seg & 1, TL::col_s(rnd & 1, slot));
            if (slot == kRound - 1 || last) {
                commit(kBarSFull0 + (rnd & 1));
                if (last)
                    commit(kBarQEmpty0 + (seg & 1));
                // This round's S^T is queued; now the PV products of the previous round.
                if (have_prev && !(ok = finish_round(prev_rnd, prev_c0, prev_nk, prev_first, prev_seg)))
                    break;
                have_prev = true;
                prev_rnd = rnd;
                prev_c0 = cur_c0;
                prev_nk = c - cur_c0 + 1;
                prev_first = cur_first;
                prev_seg = seg;
                slot = 0;
            } else {
                ++slot;
            }
            ++c;
            if (++local == cpp && g + 1 < g_end) {
                pos = locate(g + 1);
                local = pos.local;
                cpp = pos.cpp;
            }
        }
        if (ok && have_prev)
            ok = finish_round(prev_rnd, prev_c0, prev_nk, prev_first, prev_seg);
        commit(kBarDrain);
        if (!wait_drain(BAR(kBarDrain), 0, kWaitLimitNs) && leader) {
            *abort_flag = 1;
            atomicExch(p.status, kSiteDecodeConsumer);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- softmax and epilogue
        const int i = threadIdx.x;  // TMEM lane: key i of a chunk in S^T, dim i in O^T
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        const uint32_t tS = tmem + lane_base;
        const uint32_t tO = tmem + lane_base + kColO;
        constexpr int n_out = G * kD;
        if constexpr (kPaged) {
            // A sequence with no keys has nothing to attend to: O = 0 and LSE = -inf, written by
            // CTA (b mod P) since no unit of work names it.
            for (int b = cta; b < p.B; b += p.ctas) {
                if (batch_len[b] != 0)
                    continue;
                for (int h = 0; h < p.Hq; ++h) {
                    p.o[b * p.o_sb + h * p.o_sh + i] = __float2bfloat16_rn(0.f);
                    if (i == 0)
                        p.lse[static_cast<size_t>(b) * p.Hq + h] = -INFINITY;
                }
            }
        }
        bool ok = true;
        int c = 0, n_deferred = 0, sg = 0, rnd = 0;  // chunks, deferred pairs, segments, rounds so far
        for (long long g = g_begin; g < g_end;) {
            const UnitPos pos = locate(g);
            const long long pair = pos.pair;
            const int local0 = pos.local;
            const long long seg_end = min(g_end, pos.pair_start + pos.cpp);
            const int n_chunks = static_cast<int>(seg_end - g);
            const bool whole_pair = (local0 == 0) && (seg_end == pos.pair_start + pos.cpp);
            const int bk = static_cast<int>(pair / p.head_groups);
            const int b = bk / p.Hkv;
            const int h0 = (bk % p.Hkv) * p.group + static_cast<int>(pair % p.head_groups) * G;
            const int seq_len = kPaged ? batch_len[b] : p.Skv;

            // Factor from a score to log2 units, per head: the softmax scale times log2(e), and with
            // the e4m3 cache also 2^-e for the power of two the producer folded into that head's
            // Q^T parts (k_scale is folded into Q^T as well). v_coef: V's coefficient for dim i.
            float sl2[G];
            float v_coef = 1.f;
#pragma unroll
            for (int h = 0; h < G; ++h)
                sl2[h] = p.scale_log2;
            if constexpr (kFp8) {
                const int qs = sg & 1;
                const bool okq = mbar_wait(BAR(kBarQFull0 + qs), static_cast<uint32_t>(sg >> 1) & 1u, abort_flag,
                                           p.status, kSiteDecodeConsumer);
                if (okq) {
#pragma unroll
                    for (int h = 0; h < G; ++h)
                        sl2[h] = q_scale[qs * kN + h];
                }
                mbar_arrive(BAR(kBarQScFree0 + qs));
                ok = ok && okq;
                v_coef = p.v_scale[static_cast<size_t>(bk % p.Hkv) * kD + i];
                ++sg;
            }
            float m[G], l[G], lpv[G];
#pragma unroll
            for (int h = 0; h < G; ++h) {
                m[h] = -INFINITY;
                l[h] = 0.f;
                lpv[h] = 0.f;
            }
            const int n_rounds = (n_chunks + kRound - 1) / kRound;
            for (int jr = 0; jr < n_rounds; ++jr) {
                const int nk = min(kRound, n_chunks - jr * kRound);  // chunks in this round
                const int rp = rnd & 1;
                // Agreed by the warp: it gates the warp-collective TMEM loads.
                const bool okw = __all_sync(0xffffffffu, mbar_wait(BAR(kBarSFull0 + rp), static_cast<uint32_t>(rnd >> 1) & 1u,
                                                                   abort_flag, p.status, kSiteDecodeConsumer));
                float x[kRound][G];
#pragma unroll
                for (int sl = 0; sl < kRound; ++sl)
#pragma unroll
                    for (int h = 0; h < G; ++h)
                        x[sl][h] = -INFINITY;
                if (okw) {
                    tc_fence_after_sync();
#pragma unroll
                    for (int sl = 0; sl < kRound; ++sl) {
                        if (sl < nk) {
                            uint32_t r[16];
                            tmem_ld16_wait(tS + TL::col_s(rp, sl), r);
                            if constexpr (kFp8) {
#pragma unroll
                                for (int t = 1; t < TL::kParts; ++t) {
                                    uint32_t rt[16];
                                    tmem_ld16_wait(tS + TL::col_s(rp, sl) + 16u * t, rt);
#pragma unroll
                                    for (int h = 0; h < G; ++h)
                                        r[h] = __float_as_uint(__uint_as_float(r[h]) + __uint_as_float(rt[h]));
                                }
                            }
                            const bool valid = (local0 + jr * kRound + sl) * kCK + i < seq_len;
#pragma unroll
                            for (int h = 0; h < G; ++h)
                                x[sl][h] = valid ? __uint_as_float(r[h]) * sl2[h] : -INFINITY;
                        }
                    }
                }
                // After the first round the exact round max is only needed when some key exceeds the
                // reference max by the threshold: one counting barrier decides (and also catches a
                // wait that ran out); only then do the warps exchange their maxima.
                bool full = (jr == 0);
                if (!full) {
                    bool need = !(okw && ok);
#pragma unroll
                    for (int sl = 0; sl < kRound; ++sl)
#pragma unroll
                        for (int h = 0; h < G; ++h)
                            need = need || (x[sl][h] > m[h] + L::kRescaleThreshold);
                    full = bar_popc(kBarSoftmax, kSoftmaxThreads, need) != 0;
                }
                bool rescale = false;
                float cmax[G];
                if (full) {
                    if (okw) {
#pragma unroll
                        for (int h = 0; h < G; ++h) {
                            float v = x[0][h];
#pragma unroll
                            for (int sl = 1; sl < kRound; ++sl)
                                v = fmaxf(v, x[sl][h]);
#pragma unroll
                            for (int o = 16; o > 0; o >>= 1)
                                v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
                            if (lane == 0)
                                red_max[(rp * 4 + warp) * kN + h] = v;
                        }
                    }
                    // This barrier both exchanges the warps' maxima and agrees on carrying on.
                    if (!(ok = bar_and(kBarSoftmax, kSoftmaxThreads, okw && ok)))
                        break;
                    const float *rm = red_max + rp * 4 * kN;
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        cmax[h] = fmaxf(fmaxf(rm[h], rm[kN + h]), fmaxf(rm[2 * kN + h], rm[3 * kN + h]));
                        rescale = rescale || (cmax[h] > m[h] + L::kRescaleThreshold);
                    }
                }
                if (jr == 0) {
#pragma unroll
                    for (int h = 0; h < G; ++h)
                        m[h] = cmax[h];  // the round holds at least one key, so this is finite
                } else if (rescale) {
                    // The same values in every thread, so every thread takes this branch. O^T of the
                    // previous round must be complete before it is scaled.
                    float alpha[G];
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const float mn = fmaxf(m[h], cmax[h]);
                        alpha[h] = ex2(m[h] - mn);
                        m[h] = mn;
                        l[h] *= alpha[h];
                        lpv[h] *= alpha[h];
                    }
                    if (__all_sync(0xffffffffu, mbar_wait(BAR(kBarODone0 + ((rnd - 1) & 1)),
                                                          static_cast<uint32_t>((rnd - 1) >> 1) & 1u, abort_flag,
                                                          p.status, kSiteDecodeConsumer))) {
                        tc_fence_after_sync();
#pragma unroll
                        for (int t = 0; t < TL::kParts; ++t) {
                            uint32_t ov[16];
                            tmem_ld16_wait(tO + 16u * t, ov);
#pragma unroll
                            for (int h = 0; h < G; ++h)
                                ov[h] = __float_as_uint(__uint_as_float(ov[h]) * alpha[h]);
                            tmem_st16_wait(tO + 16u * t, ov);
                        }
                    } else {
                        ok = false;
                    }
                }
                // Weights, both running sums, and P^T (row h, column i) of each chunk of the round for
                // its PV product. P^T is K-major with the 128-byte swizzle: key i sits in half i / 64
                // of row h, in 16-byte unit ((i % 64) / 8) XOR (h % 8).
#pragma unroll
                for (int sl = 0; sl < kRound; ++sl) {
                    if (sl >= nk)
                        break;
                    if constexpr (kFp8) {
                        // e4m3 cache: the weight times 16 as three e4m3 parts, each in its own 16 x 128-byte
                        // tile: key i is byte (i % 16) of 16-byte unit (i / 16) XOR (h % 8) in row h. lpv sums
                        // what the PV product uses (in units of 1/16, like O^T).
                        uint8_t *pbuf = smem + kOffP + (rp * kRound + sl) * kSmallBytes;
                        auto off_of = [&](int h) { return (h >> 3) * 1024 + (h & 7) * 128 + ((((i >> 4) ^ (h & 7)) << 4) | (i & 15)); };
#pragma unroll
                        for (int h = 0; h < G; h += 2) {  // two heads per conversion
                            constexpr bool kPair = G > 1;
                            const float pa = ex2(x[sl][h] - m[h]);
                            const float pb = kPair ? ex2(x[sl][h + (kPair ? 1 : 0)] - m[h + (kPair ? 1 : 0)]) : 0.f;
                            float wa = pa * L::kPScale, wb = pb * L::kPScale;
                            const float ua = wa, ub = wb;
#pragma unroll
                            for (int t = 0; t < 3; ++t) {
                                const uint32_t cd = e4m3x2(wa, wb);
                                const float2 v = e4m3x2_value(cd);
                                wa -= v.x;
                                wb -= v.y;
                                pbuf[t * kSmallHalf + off_of(h)] = static_cast<uint8_t>(cd & 0xffu);
                                if (kPair)
                                    pbuf[t * kSmallHalf + off_of(h + 1)] = static_cast<uint8_t>((cd >> 8) & 0xffu);
                            }
                            // The parts' sum is the weight minus what is left over (exact: it needs ~12 bits).
                            l[h] += pa;
                            lpv[h] += ua - wa;
                            if (kPair) {
                                l[h + (kPair ? 1 : 0)] += pb;
                                lpv[h + (kPair ? 1 : 0)] += ub - wb;
                            }
                        }
                    } else {
                        uint8_t *pbuf = smem + kOffP + (rp * kRound + sl) * kSmallBytes + (i >> 6) * kSmallHalf;
                        const int kk = i & 63;
#pragma unroll
                        for (int h = 0; h < G; ++h) {
                            const float pe = ex2(x[sl][h] - m[h]);
                            l[h] += pe;
                            const __nv_bfloat16 pb = __float2bfloat16_rn(pe);
                            lpv[h] += __bfloat162float(pb);
                            const int off = (h >> 3) * 1024 + (h & 7) * 128 + ((((kk >> 3) ^ (h & 7)) << 4) | ((kk & 7) << 1));
                            *reinterpret_cast<__nv_bfloat16 *>(pbuf + off) = pb;
                        }
                    }
                    if constexpr (kPaged) {
                        // Rows past the sequence's length in its last page hold whatever the cache holds
                        // there; their weights are 0, but 0 * NaN is not, so zero them before the PV product.
                        if ((local0 + jr * kRound + sl) * kCK + i >= seq_len) {
                            uint4 *vrow = reinterpret_cast<uint4 *>(smem + kOffRing + ((c + sl) % kStages) * kStageBytes +
                                                                    kTileBytes + i * 128);
#pragma unroll
                            for (int hf = 0; hf < L::kBoxCols; ++hf)
#pragma unroll
                                for (int u = 0; u < 8; ++u)
                                    vrow[hf * (kHalfBytes / 16) + u] = make_uint4(0u, 0u, 0u, 0u);
                        }
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before_sync();
                mbar_arrive(BAR(kBarPFull0 + rp));
                c += nk;
                ++rnd;
            }
            if (!ok)
                break;

            // ------------------------------------------------ end of segment
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float a = l[h], q = lpv[h];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    a += __shfl_xor_sync(0xffffffffu, a, o);
                    q += __shfl_xor_sync(0xffffffffu, q, o);
                }
                if (lane == 0) {
                    red_sum[(warp * kN + h) * 2] = a;
                    red_sum[(warp * kN + h) * 2 + 1] = q;
                }
            }
            const bool okw = mbar_wait(BAR(kBarODone0 + ((rnd - 1) & 1)), static_cast<uint32_t>((rnd - 1) >> 1) & 1u,
                                       abort_flag, p.status, kSiteDecodeConsumer);
            if (!(ok = bar_and(kBarSoftmax, kSoftmaxThreads, okw && ok)))
                break;
            tc_fence_after_sync();
            uint32_t ov[16];
            tmem_ld16_wait(tO, ov);
#pragma unroll
            for (int t = 1; t < TL::kParts; ++t) {
                uint32_t ot[16];
                tmem_ld16_wait(tO + 16u * t, ot);
#pragma unroll
                for (int h = 0; h < G; ++h)
                    ov[h] = __float_as_uint(__uint_as_float(ov[h]) + __uint_as_float(ot[h]));
            }
            tc_fence_before_sync();
            mbar_arrive(BAR(kBarOFree));  // the next segment may overwrite O^T

            // A CTA writes at most two partials: of its first segment (slot 0) and of its last one
            // (slot 1); the merging CTA finds them the same way (see below).
            const int which = (g == g_begin) ? 0 : 1;
            float *slot_base = p.ws + (static_cast<size_t>(cta) * 2 + which) * (n_out + G);
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float L = 0.f, LPV = 0.f;
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    L += red_sum[(w * kN + h) * 2];
                    LPV += red_sum[(w * kN + h) * 2 + 1];
                }
                const float o = __uint_as_float(ov[h]) / LPV * v_coef;
                const size_t bh = static_cast<size_t>(b) * p.Hq + h0 + h;
                if (whole_pair) {
                    p.o[b * p.o_sb + (h0 + h) * p.o_sh + i] = __float2bfloat16_rn(o);
                    if (i == h)
                        p.lse[bh] = (m[h] + log2f(L)) * kLn2;
                } else {
                    slot_base[h * kD + i] = o;
                    if (i == h)
                        slot_base[n_out + h] = m[h] + log2f(L);
                }
            }
            if (!whole_pair) {
                // Signalled once the whole range is streamed (below): only the first and the last
                // segment of a range can be a piece of a shared pair.
                if (i == 0)
                    deferred_pair[n_deferred] = pair;
                ++n_deferred;
            }
            g = seg_end;
        }

        // ---------------------------------------------------------------- shared pairs: the last CTA merges
        if (ok) {
            int n_def = 0;
            if (i == 0) {
                n_def = n_deferred;
                if (n_def > 0)
                    __threadfence();  // publish this CTA's partials before the counters move
                for (int k = 0; k < n_def; ++k) {
                    // The pair's contributors: the CTAs from the one holding its first unit to the
                    // one holding its last, except those with an empty range (fewer units than CTAs).
                    const long long pr = deferred_pair[k];
                    int pr_cpp = 0;
                    const long long pr_start = pair_first_unit(pr, &pr_cpp);
                    const int first = cta_of_unit(pr_start, total, p.ctas);
                    const int last = cta_of_unit(pr_start + pr_cpp - 1, total, p.ctas);
                    int n_contrib = 0;
                    for (int cc = first; cc <= last; ++cc)
                        n_contrib += (range_start(cc, total, p.ctas) < range_start(cc + 1, total, p.ctas)) ? 1 : 0;
                    deferred_first[k] = first;
                    const int prev = atomicAdd(&p.counters[pr], 1);
                    last_flag[k] = (prev == n_contrib - 1) ? last - first + 1 : 0;
                }
                last_flag[2] = n_def;
            }
            bar_and(kBarSoftmax, kSoftmaxThreads, true);
            n_def = last_flag[2];
            for (int k = 0; k < n_def; ++k) {
                const int n_contrib = last_flag[k];
                if (n_contrib == 0)
                    continue;
                __threadfence();
                const long long pr = deferred_pair[k];
                const int bk = static_cast<int>(pr / p.head_groups);
                const int b = bk / p.Hkv;
                const int h0 = (bk % p.Hkv) * p.group + static_cast<int>(pr % p.head_groups) * G;
                // n_contrib here is the span of CTAs (first .. first + span - 1); a contributor whose
                // range starts inside the pair wrote its first segment (slot 0), the one whose range
                // started before it wrote its last segment (slot 1).
                const int first = deferred_first[k];
                int pr_cpp = 0;
                const long long pr_start = pair_first_unit(pr, &pr_cpp);
                auto slot_of = [&](int cc) -> const float * {
                    const int which = (range_start(cc, total, p.ctas) >= pr_start) ? 0 : 1;
                    return p.ws + (static_cast<size_t>(cc) * 2 + which) * (n_out + G);
                };
                auto contributes = [&](int cc) {
                    return range_start(cc, total, p.ctas) < range_start(cc + 1, total, p.ctas);
                };
                for (int idx = i; idx < n_out; idx += kSoftmaxThreads) {
                    const int h = idx / kD;
                    const int d = idx % kD;
                    float M = -INFINITY;
                    for (int cc = first; cc < first + n_contrib; ++cc)
                        if (contributes(cc))
                            M = fmaxf(M, __ldcg(slot_of(cc) + n_out + h));
                    float W = 0.f, O = 0.f;
                    for (int cc = first; cc < first + n_contrib; ++cc) {
                        if (!contributes(cc))
                            continue;
                        const float *sb = slot_of(cc);
                        const float w = ex2(__ldcg(sb + n_out + h) - M);
                        W += w;
                        O = fmaf(w, __ldcg(sb + idx), O);
                    }
                    const size_t bh = static_cast<size_t>(b) * p.Hq + h0 + h;
                    p.o[b * p.o_sb + (h0 + h) * p.o_sh + d] = __float2bfloat16_rn(O / W);
                    if (d == 0)
                        p.lse[bh] = (M + log2f(W)) * kLn2;
                }
                if (i == 0)
                    atomicExch(&p.counters[pr], 0);  // ready for the next call
            }
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, TmemLay<kFp8>::kCols);
    }
#undef BAR
}

template <int G, bool kPaged, bool kFp8>
cudaError_t prepare_g(int *ctas_per_sm)
{
    static int cached_per_dev[kMaxDevices] = {};  // per device: attributes apply to the current one
    constexpr int kSmem = Lay<kFp8>::kSmem;
    const int dev = current_device_index();
    if (dev < 0)
        return cudaErrorInvalidDevice;
    int &cached = cached_per_dev[dev];
    if (cached == 0) {
        cudaError_t e = cudaFuncSetAttribute(decode_tc_kernel<G, kPaged, kFp8>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
        int n = 0;
        if (e == cudaSuccess)
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_tc_kernel<G, kPaged, kFp8>, kThreads, kSmem);
        if (e != cudaSuccess)
            return e;
        cached = n > 0 ? n : 1;
    }
    if (ctas_per_sm)
        *ctas_per_sm = cached;
    return cudaSuccess;
}

template <int G, bool kPaged, bool kFp8>
cudaError_t launch_g(const DecodeArgs &a, cudaStream_t stream)
{
    cudaError_t e = prepare_g<G, kPaged, kFp8>(nullptr);
    if (e != cudaSuccess)
        return e;
    auto encode = get_encode_fn();
    if (!encode)
        return cudaErrorInitializationError;
    int err = 0;
    CUtensorMap tq, tk, tv;
    // q: heads as the rows of a (dim, head, 1, batch) map, boxes of 16 heads; k and v: (dim, key,
    // kv head, batch) with the caller's strides, or, paged, (dim, slot, kv head, page) over
    // [num_pages][Hkv][page_size][D], read in boxes of min(page_size, 128) rows and 128 bytes of D
    // (64 bf16 or 128 e4m3 elements).
    const TensorStrides qs = a.strided ? a.qs : TensorStrides{static_cast<long long>(a.Hq) * kD, kD, kD};
    const int box_rows = kPaged ? (a.page_size < kCK ? a.page_size : kCK) : kCK;
    if (!make_map4(encode, &tq, a.q, 2, kD, a.Hq, 1, a.B, Strides{qs.b, qs.b, qs.h}, 64, kN,
                   CU_TENSOR_MAP_SWIZZLE_128B, &err))
        return cudaErrorInvalidValue;
    constexpr int kElem = kFp8 ? 1 : 2;
    constexpr int kBoxInner = kFp8 ? 128 : 64;
    Strides kst, vst;
    if (kPaged) {
        kst = vst = Strides{static_cast<long long>(a.Hkv) * a.page_size * kD, static_cast<long long>(a.page_size) * kD, kD};
    } else if (a.strided) {
        kst = Strides{a.ks.b, a.ks.h, a.ks.s};
        vst = Strides{a.vs.b, a.vs.h, a.vs.s};
    } else {
        kst = vst = contiguous_strides(a.Hkv, a.Skv, kD);
    }
    const int kv_rows = kPaged ? a.page_size : a.Skv;
    const int kv_outer = kPaged ? a.num_pages : a.B;
    if (!make_map4(encode, &tk, a.k, kElem, kD, kv_rows, a.Hkv, kv_outer, kst, kBoxInner, box_rows,
                   CU_TENSOR_MAP_SWIZZLE_128B, &err) ||
        !make_map4(encode, &tv, a.v, kElem, kD, kv_rows, a.Hkv, kv_outer, vst, kBoxInner, box_rows,
                   CU_TENSOR_MAP_SWIZZLE_128B, &err))
        return cudaErrorInvalidValue;
    const DecodePlan &pl = a.plan;
    TcParams p;
    p.o = static_cast<__nv_bfloat16 *>(a.o);
    p.o_sb = a.strided ? a.os.b : static_cast<long long>(a.Hq) * kD;
    p.o_sh = a.strided ? a.os.h : kD;
    p.q_sb = qs.b;
    p.q_sh = qs.h;
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
    p.total = pl.total;
    p.scale_log2 = a.scale * kLog2e;
    p.seq_lens = a.seq_lens;
    p.block_table = a.block_table;
    p.B = a.B;
    p.num_pages = a.num_pages;
    p.page_size = a.page_size;
    p.pages_per_seq = a.pages_per_seq;
    p.max_seq_len = a.max_seq_len;
    p.q = static_cast<const __nv_bfloat16 *>(a.q);
    p.k_scale = a.k_scale;
    p.v_scale = a.v_scale;
    decode_tc_kernel<G, kPaged, kFp8>
        <<<static_cast<unsigned>(pl.ctas), kThreads, Lay<kFp8>::kSmem, stream>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

template <int G>
cudaError_t dispatch_g(const DecodeArgs *a, cudaStream_t stream, int *ctas_per_sm, bool fp8 = false)
{
    if (!a)
        return fp8 ? prepare_g<G, false, true>(ctas_per_sm) : prepare_g<G, false, false>(ctas_per_sm);
    if (a->fp8)
        return a->seq_lens ? launch_g<G, true, true>(*a, stream) : launch_g<G, false, true>(*a, stream);
    return a->seq_lens ? launch_g<G, true, false>(*a, stream) : launch_g<G, false, false>(*a, stream);
}

cudaError_t dispatch_tc(int G, const DecodeArgs *a, cudaStream_t stream, int *ctas_per_sm, bool fp8 = false)
{
    switch (G) {
    case 1:
        return dispatch_g<1>(a, stream, ctas_per_sm, fp8);
    case 2:
        return dispatch_g<2>(a, stream, ctas_per_sm, fp8);
    case 4:
        return dispatch_g<4>(a, stream, ctas_per_sm, fp8);
    case 8:
        return dispatch_g<8>(a, stream, ctas_per_sm, fp8);
    case 16:
        return dispatch_g<16>(a, stream, ctas_per_sm, fp8);
    default:
        return cudaErrorInvalidValue;
    }
}

}  // namespace

int decode_tc_heads_per_pair(int group)
{
    // Largest power of two that divides the group size, at most the MMA's N of 16.
    int g = 1;
    while (g < kN && group % (2 * g) == 0)
        g *= 2;
    return g;
}

int decode_tc_chunk_keys() { return kCK; }

cudaError_t decode_tc_ctas_per_sm(int G, bool fp8, int *ctas_per_sm)
{
    return dispatch_tc(G, nullptr, nullptr, ctas_per_sm, fp8);
}

cudaError_t launch_decode_tc(const DecodeArgs &a, cudaStream_t stream) { return dispatch_tc(a.plan.G, &a, stream, nullptr); }

size_t decode_tc_partial_floats(int G, int ctas) { return static_cast<size_t>(2) * ctas * (static_cast<size_t>(G) * kD + G); }

cudaError_t decode_plan_paged(int B, int Hq, int Hkv, int max_seq_len, int requested_ctas, int sm_count,
                              DecodePlan *plan, bool fp8)
{
    DecodePlan pl;
    const int group = Hq / Hkv;
    pl.G = decode_tc_heads_per_pair(group);
    pl.head_groups = group / pl.G;
    pl.pairs = static_cast<long long>(B) * Hkv * pl.head_groups;
    pl.ck = kCK;
    pl.cpp = (max_seq_len + kCK - 1) / kCK;  // an upper bound: lengths are read on the device
    pl.total = 0;                            // computed by each CTA from the lengths
    long long ctas = requested_ctas;
    if (ctas <= 0) {
        int per_sm = 1;
        const cudaError_t e = fp8 ? prepare_g<1, true, true>(&per_sm) : prepare_g<1, true, false>(&per_sm);
        if (e != cudaSuccess)
            return e;
        // As for the dense cache: one CTA per pair when the pairs alone fill most of the GPU
        // (measured faster than sharing pairs among all SMs), else one CTA per resident slot.
        const long long slots = static_cast<long long>(sm_count) * per_sm;
        ctas = (pl.pairs <= slots && 4 * pl.pairs >= 3 * slots) ? pl.pairs : slots;
    }
    if (ctas > (1LL << 22))
        return cudaErrorInvalidValue;
    pl.ctas = static_cast<int>(ctas);
    pl.max_contrib = 0;  // unused by this kernel: partials are kept per CTA
    pl.partial_floats = decode_tc_partial_floats(pl.G, pl.ctas);
    *plan = pl;
    return cudaSuccess;
}

}  // namespace attn_b200
