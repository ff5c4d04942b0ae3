/*
 * prefill_fp8_sm100.cu — causal prefill (any Sq <= Skv) over a K/V cache stored as e4m3 codes with
 * fp32 per-(kv head, channel) coefficients, on sm_100a: the tensor core reads the cache's codes
 * as they are (tcgen05.mma kind::f8f6f4, fp32 accumulation in tensor memory).
 *
 * What it computes (the dequantised definition): with k[b,g,j,d] = e4m3(k8) * k_scale[g][d] and
 * v[b,g,j,d] = e4m3(v8) * v_scale[g][d], the attention of attn_fwd over those values: the causal
 * mask aligned to the last Sq keys, o and lse as attn_fwd.
 *
 * One CTA per (128-row query tile, query head, batch), two CTAs per SM (their chains interleave on
 * the SM's tensor core), 192 threads: warps 0-3 one query row each (thread = row = TMEM lane),
 * warp 4 TMA producer, warp 5 TMEM allocator and MMA issuer. Per CTA:
 *   set-up  each row thread forms x = q * k_scale (fp32), scales it by the power of two 2^e that
 *           puts max|x| in (224, 448] (the top of the e4m3 range), and splits it into three e4m3
 *           parts (each the rounding of what the previous parts left; about 12 significant bits),
 *           K-major with the 128-byte swizzle: A operands of the score product;
 *   per KV tile of 128 keys (K and V tiles of 16 KB each, two stages):
 *     S = [Q_1 | Q_2 | Q_3] [K | K | K]^T   12 instructions of M = N = 128, K = 32 into TMEM
 *     softmax  thread = row: S * 2^-e * scale * log2(e), causal mask, row max in two passes over
 *              the tile (the reference max moves only when it grows by more than 4, then O is
 *              rescaled), weights 2^(s - m) times 16 split into two e4m3 parts (about 8
 *              significant bits, the precision the bf16 path gives P; the split runs in f16x2
 *              arithmetic, two weights per instruction) and written back into TMEM
 *              over the S columns already read (part t of keys 32c.. in columns 16c + 8t: never a
 *              column the pass has not read yet);
 *     O += [P_1 | P_2] [V; V]                8 instructions, A = the parts from TMEM, B = V read
 *              MN-major (one 128-byte atom spans the 128 dims). Three parts for the weights
 *              measured 12-15% slower for no accuracy the tolerance needs;
 *   epilogue O * v_scale / (sum of the parts' values), LSE from the sum of the exact weights.
 *
 * TMEM: 256 columns per CTA, S (then P) in [0, 128), O in [128, 256). The MMAs of one thread run
 * in issue order, so tile j's PV product has read P before tile j+1's S product overwrites it.
 *
 * Sources (page title, section): FP8 storage with higher-precision accumulation — "MLA 矩阵乘法吸收
 * 的数值稳定性治理", §五; a coefficient per feature channel — same page, §二.1; the causal mask
 * aligned to the last Sq keys — "第11节：Attention 实现（Flash vs Fallback）", §3; online softmax
 * with a lazy reference max and the LSE — "AI Infra 入门：RMSNorm、Softmax、Causal Mask、Sampling
 * 的数学与底层优化", §2–§3.
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

constexpr int kD = 128;
constexpr int kBM = 128;  // query rows per CTA (TMEM lanes)
constexpr int kBN = 128;  // keys per KV tile
constexpr int kThreads = 192;
constexpr int kWarpTma = 4;
constexpr int kWarpMma = 5;
constexpr int kStages = 2;
constexpr int kParts = 3;   // e4m3 parts of q * k_scale (about 12 significant bits)
constexpr int kPParts = 2;  // e4m3 parts of the weights (about 8 significant bits, as bf16 P)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kThreshold = 4.0f;  // log2 units; weights stay below 2^4 * 16 = 256 < 448
constexpr float kPScale = 16.0f;

constexpr int kPartBytes = kBM * 128;  // one e4m3 part of the query tile: 128 rows x 128 bytes
constexpr int kTileBytes = kBN * 128;  // one e4m3 K or V tile
constexpr int kOffQ = 0;
constexpr int kOffRing = kOffQ + kParts * kPartBytes;  // [stage]: K tile, then V tile
constexpr int kStageBytes = 2 * kTileBytes;
constexpr int kOffBar = kOffRing + kStages * kStageBytes;
enum Fp8Bar : int {
    kBarFull0 = 0,                  // [stage] K and V tiles landed
    kBarEmpty0 = kBarFull0 + kStages,  // [stage] both products done with the stage
    kBarSFull = kBarEmpty0 + kStages,  // S of the current tile in TMEM
    kBarPFull = kBarSFull + 1,         // P parts in TMEM (128 arrivals)
    kBarODone = kBarPFull + 1,         // the tile's PV product done
    kBarDrain = kBarODone + 1,         // every product issued has completed
    kNumBars = kBarDrain + 1,
};
constexpr int kOffMisc = kOffBar + kNumBars * 8;  // TMEM slot, abort flag
constexpr int kSmem = kOffMisc + 64;  // the dynamic window starts 1024-aligned (no static smem)
static_assert(kSmem <= 113 * 1024, "two CTAs per SM");
constexpr uint32_t kTmemCols = 256, kColS = 0, kColO = 128;

struct Fp8PrefillParams {
    const __nv_bfloat16 *q;
    const float *k_scale, *v_scale;  // [Hkv][D]
    __nv_bfloat16 *o;
    float *lse;
    int *status;
    int B, Hq, Hkv, Sq, Skv, group, offset, causal, n_qtiles;
    float scale_log2;  // scale * log2(e)
};

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Codes of (a, b) as e4m3 (round to nearest even, saturating), a in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float a, float b)
{
    return __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
}

__device__ __forceinline__ float2 e4m3x2_value(uint32_t codes)
{
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(codes), __NV_E4M3);
    return __half22float2(__half2(h));
}

// One split step over four values: their codes (value u in byte u), and x -= the codes' values
// (exact: a value and its 3-bit rounding lie within a factor of two of each other).
__device__ __forceinline__ uint32_t split4(float (&x)[4])
{
    const uint32_t lo = e4m3x2(x[0], x[1]), hi = e4m3x2(x[2], x[3]);
    const float2 vl = e4m3x2_value(lo), vh = e4m3x2_value(hi);
    x[0] -= vl.x;
    x[1] -= vl.y;
    x[2] -= vh.x;
    x[3] -= vh.y;
    return lo | (hi << 16);
}

// The power of two e that brings mx (> 0) into (224, 448]; 0 for mx = 0; clamped to [-100, 100].
__device__ __forceinline__ int scale_exponent(float mx)
{
    if (!(mx > 0.f))
        return 0;
    const uint32_t bits = __float_as_uint(mx);
    const int E = static_cast<int>((bits >> 23) & 255u) - 127;
    const float mant = __uint_as_float((bits & 0x007fffffu) | 0x3f800000u);  // in [1, 2)
    const int e = (mant <= 1.75f ? 8 : 7) - E;
    return min(max(e, -100), 100);
}

__device__ __forceinline__ float exp2_int(int e) { return __uint_as_float(static_cast<uint32_t>(e + 127) << 23); }

// Warp-collective TMEM store of 32 lanes x 8 consecutive columns, without the wait.
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem] with 8-bit floating-point operands: A (M x K, K-major) in tensor
// memory, row i in lane i, four elements per 32-bit column (element 4c + u in byte u of column c).
__device__ __forceinline__ void tc_mma_f8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
                 "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
                 : "memory");
}

__device__ __forceinline__ bool wait_drain(uint32_t bar, uint32_t parity, uint64_t limit_ns)
{
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > limit_ns)
            return false;
    }
    return true;
}

// acc + lo + hi for the two f16 values packed in w, each added with fp32 accumulation (mixed-
// precision adds: no separate widening of the f16 halves).
__device__ __forceinline__ float add_f16x2(float acc, uint32_t w)
{
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\t"
        "add.rn.f32.f16 %0, lo, %0;\n\tadd.rn.f32.f16 %0, hi, %0;\n\t}"
        : "+f"(acc)
        : "r"(w));
    return acc;
}

// Three-input maximum (one instruction on sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

__global__ void __launch_bounds__(kThreads, 2)
    prefill_fp8_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                       const Fp8PrefillParams p)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t s_base = smem_u32(smem);
    const uint32_t bar0 = s_base + kOffBar;
#define BAR(i) (bar0 + 8u * static_cast<uint32_t>(i))
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffMisc + 4);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (s_base & 1023u) {  // the swizzled tiles need the 1024-byte alignment the window starts with
        if (threadIdx.x == 0)
            atomicExch(p.status, kSiteFp8Prefill);
        return;
    }

    // Work: query tiles slowest and heaviest first (the last rows see the most keys), so that the
    // short tiles fill in behind the long ones; then heads, then batch.
    const int heads = p.Hq * p.B;
    const int qt = p.n_qtiles - 1 - static_cast<int>(blockIdx.x / heads);
    const int hb = static_cast<int>(blockIdx.x % heads);
    const int h = hb % p.Hq;
    const int b = hb / p.Hq;
    const int kvh = h / p.group;
    const int q0 = qt * kBM;
    const int last_key = p.causal ? min(p.Skv - 1, q0 + kBM - 1 + p.offset) : p.Skv - 1;
    const int n_tiles = last_key / kBN + 1;

    float row_factor = 0.f;  // score units per unit of the part sum: 2^-e * scale * log2(e)
    if (warp < 4) {
        // Q parts of this thread's row (zeros past Sq).
        const int r = threadIdx.x;
        const int qi = q0 + r;
        const bool valid = qi < p.Sq;
        const __nv_bfloat16 *qrow = p.q + ((static_cast<size_t>(b) * p.Hq + h) * p.Sq + (valid ? qi : 0)) * kD;
        const float4 *ks4 = reinterpret_cast<const float4 *>(p.k_scale + static_cast<size_t>(kvh) * kD);
        // The row (256 bytes) is loaded once, all sixteen 16-byte loads in flight together; x = q *
        // k_scale is then formed 16 dims at a time from it (two passes over the row).
        uint4 qr[kD / 8];
        {
            const uint4 *src = reinterpret_cast<const uint4 *>(qrow);
#pragma unroll
            for (int t = 0; t < kD / 8; ++t)
                qr[t] = valid ? src[t] : make_uint4(0u, 0u, 0u, 0u);
        }
        auto load16 = [&](int c, float (&x)[16]) {
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const uint4 raw = qr[2 * c + hf];
                const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
                const float4 sa = ks4[4 * c + 2 * hf], sb = ks4[4 * c + 2 * hf + 1];
                const float sc[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    x[8 * hf + 2 * u] = __uint_as_float(w[u] << 16) * sc[2 * u];
                    x[8 * hf + 2 * u + 1] = __uint_as_float(w[u] & 0xffff0000u) * sc[2 * u + 1];
                }
            }
        };
        float mx = 0.f;
#pragma unroll
        for (int c = 0; c < kD / 16; ++c) {
            float x[16];
            load16(c, x);
#pragma unroll
            for (int u = 0; u < 16; ++u)
                mx = fmaxf(mx, fabsf(x[u]));
        }
        const int e = scale_exponent(mx);
        const float f = exp2_int(e);
        row_factor = p.scale_log2 * exp2_int(-e);
        // Part pt of row r: 128 bytes, 16-byte unit c (dims 16c .. 16c + 15) at ((c ^ (r % 8)) << 4)
        // (K-major, 128-byte swizzle).
#pragma unroll
        for (int c = 0; c < kD / 16; ++c) {
            float x[16];
            load16(c, x);
            uint32_t wd[kParts][4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                float v4[4] = {x[4 * u] * f, x[4 * u + 1] * f, x[4 * u + 2] * f, x[4 * u + 3] * f};
#pragma unroll
                for (int pt = 0; pt < kParts; ++pt)
                    wd[pt][u] = split4(v4);
            }
#pragma unroll
            for (int pt = 0; pt < kParts; ++pt)
                *reinterpret_cast<uint4 *>(smem + kOffQ + pt * kPartBytes + r * 128 + ((c ^ (r & 7)) << 4)) =
                    make_uint4(wd[pt][0], wd[pt][1], wd[pt][2], wd[pt][3]);
        }
        fence_proxy_async_smem();  // the parts are A operands of the score product
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(BAR(kBarFull0 + s), 1);
            mbar_init(BAR(kBarEmpty0 + s), 1);
        }
        mbar_init(BAR(kBarSFull), 1);
        mbar_init(BAR(kBarPFull), 128);
        mbar_init(BAR(kBarODone), 1);
        mbar_init(BAR(kBarDrain), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == kWarpTma) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            const int row = b * p.Hkv + kvh;
            int j = 0;
            for (; j < n_tiles; ++j) {
                const int st = j % kStages;
                if (!mbar_wait(BAR(kBarEmpty0 + st), (static_cast<uint32_t>(j / kStages) & 1u) ^ 1u, abort_flag, p.status,
                               kSiteFp8Prefill))
                    break;
                const uint32_t dst = s_base + kOffRing + st * kStageBytes;
                mbar_arrive_expect_tx(BAR(kBarFull0 + st), kStageBytes);
                tma_load_3d(dst, &tm_k, BAR(kBarFull0 + st), 0, j * kBN, row);
                tma_load_3d(dst + kTileBytes, &tm_v, BAR(kBarFull0 + st), 0, j * kBN, row);
            }
            if (*abort_flag)
                for (int c = (j > kStages ? j - kStages : 0); c < j; ++c)
                    wait_drain(BAR(kBarFull0 + c % kStages), static_cast<uint32_t>(c / kStages) & 1u, 100000000ull);
        }
    } else if (warp == kWarpMma) {
        // ---------------------------------------------------------------- MMA issuer
        const bool leader = elect_one();
        constexpr uint32_t kIdS = idesc_e4m3_f32_ab(kBM, kBN, false, false);  // A = Q parts, B = K tile
        constexpr uint32_t kIdO = idesc_e4m3_f32_ab(kBM, kD, false, true);    // A = P parts, B = V read MN-major
        auto commit = [&](int bar) {
            if (leader)
                tc_commit(BAR(bar));
        };
        bool ok = true;
        for (int j = 0; ok && j < n_tiles; ++j) {
            const int st = j % kStages;
            if (!(ok = mbar_wait(BAR(kBarFull0 + st), static_cast<uint32_t>(j / kStages) & 1u, abort_flag, p.status,
                                 kSiteFp8Prefill)))
                break;
            tc_fence_after_sync();
            const uint32_t sK = s_base + kOffRing + st * kStageBytes, sV = sK + kTileBytes;
            if (leader) {
                // S overwrites the previous tile's P: issued after that tile's PV product.
#pragma unroll
                for (int pt = 0; pt < kParts; ++pt)
#pragma unroll
                    for (int kk = 0; kk < kD / 32; ++kk)
                        tc_mma_f8_ss(tmem + kColS,
                                     smem_desc(s_base + kOffQ + pt * kPartBytes + kk * 32, 16, 1024, kSwizzle128B),
                                     smem_desc(sK + kk * 32, 16, 1024, kSwizzle128B), kIdS, (pt | kk) ? 1u : 0u);
            }
            commit(kBarSFull);
            if (!(ok = mbar_wait(BAR(kBarPFull), static_cast<uint32_t>(j) & 1u, abort_flag, p.status, kSiteFp8Prefill)))
                break;
            tc_fence_after_sync();
            if (leader) {
                // Part pt of keys 32 kk .. 32 kk + 31 sits in columns 16 kk + 8 pt.
#pragma unroll
                for (int pt = 0; pt < kPParts; ++pt)
#pragma unroll
                    for (int kk = 0; kk < kBN / 32; ++kk)
                        tc_mma_f8_ts(tmem + kColO, tmem + kColS + 8u * kPParts * kk + 8u * pt,
                                     smem_desc(sV + kk * 32 * 128, kTileBytes, 1024, kSwizzle128B), kIdO,
                                     (j > 0 || pt > 0 || kk > 0) ? 1u : 0u);
            }
            commit(kBarODone);
            commit(kBarEmpty0 + st);
        }
        // Every product issued completes before TMEM is released (also after an abort).
        commit(kBarDrain);
        if (!wait_drain(BAR(kBarDrain), 0, kWaitLimitNs) && leader) {
            *abort_flag = 1;
            atomicExch(p.status, kSiteFp8Prefill);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- softmax and epilogue
        const int r = threadIdx.x;  // query row within the tile == TMEM lane
        const int qi = q0 + r;
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        const uint32_t tS = tmem + lane_base + kColS, tO = tmem + lane_base + kColO;
        const int key_limit = p.causal ? min(p.Skv - 1, qi + p.offset) : p.Skv - 1;  // last visible key
        float m_ref = -INFINITY, l = 0.f, lpv = 0.f;
        bool ok = true;
        for (int j = 0; j < n_tiles; ++j) {
            // Agreed by the warp: it gates the warp-collective TMEM loads and stores.
            if (!(ok = __all_sync(0xffffffffu, mbar_wait(BAR(kBarSFull), static_cast<uint32_t>(j) & 1u, abort_flag,
                                                         p.status, kSiteFp8Prefill))))
                break;
            tc_fence_after_sync();
            const int k0 = j * kBN;
            // Every key of the tile visible to this row: no per-key mask below.
            const bool full = k0 + kBN - 1 <= key_limit;
            // Pass 1: the row max of the tile (masked keys excluded), on the raw part sums (the
            // factor to score units is positive), in eight independent chains.
            float mx8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                mx8[i] = -INFINITY;
#pragma unroll 1
            for (int c2 = 0; c2 < kBN / 64; ++c2) {
                uint32_t sra[32], srb[32];
                tmem_ld32x2_wait(tS + c2 * 64, tS + c2 * 64 + 32, sra, srb);
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const int c = 2 * c2 + hf;
                    uint32_t(&sr)[32] = hf ? srb : sra;
                    if (full) {
#pragma unroll
                        for (int u = 0; u < 32; u += 4) {
                            float &m8 = mx8[u / 4];
                            m8 = fmax3(m8, __uint_as_float(sr[u]), __uint_as_float(sr[u + 1]));
                            m8 = fmax3(m8, __uint_as_float(sr[u + 2]), __uint_as_float(sr[u + 3]));
                        }
                    } else {
#pragma unroll
                        for (int u = 0; u < 32; ++u)
                            if (k0 + c * 32 + u <= key_limit)
                                mx8[u & 7] = fmaxf(mx8[u & 7], __uint_as_float(sr[u]));
                    }
                }
            }
            const float mx =
                fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])) * row_factor;
            // The reference max: the first tile's max (finite: every row sees key 0), then moved
            // only when a tile's max exceeds it by more than the threshold; O is then rescaled once
            // the previous tile's PV product is done.
            float alpha = 1.f;
            if (j == 0) {
                m_ref = mx;
            } else if (mx > m_ref + kThreshold) {
                alpha = ex2(m_ref - mx);
                m_ref = mx;
            }
            if (__any_sync(0xffffffffu, alpha != 1.f)) {
                if (!(ok = __all_sync(0xffffffffu, mbar_wait(BAR(kBarODone), static_cast<uint32_t>(j - 1) & 1u,
                                                             abort_flag, p.status, kSiteFp8Prefill))))
                    break;
                tc_fence_after_sync();
#pragma unroll 1
                for (int c = 0; c < kD / 32; ++c) {
                    uint32_t ov[32];
                    tmem_ld32_wait(tO + c * 32, ov);
#pragma unroll
                    for (int u = 0; u < 32; ++u)
                        ov[u] = __float_as_uint(__uint_as_float(ov[u]) * alpha);
                    tmem_st32_wait(tO + c * 32, ov);
                }
                l *= alpha;
                lpv *= alpha;
            }
            // Pass 2: weights, their two e4m3 parts (x16) into TMEM over the columns already read; the
            // sums in four independent chains each.
            // The weights come out times 16 (kPScale) straight from the exponent; l is kept in those
            // units within the tile and scaled back (exactly) when it joins the running sum.
            const float m16 = m_ref - 4.0f;  // 2^4 = kPScale
            float l4[4] = {0.f, 0.f, 0.f, 0.f}, lpv4[2] = {0.f, 0.f};
#pragma unroll 1
            for (int c2 = 0; c2 < kBN / 64; ++c2) {
                uint32_t sra[32], srb[32];
                tmem_ld32x2_wait(tS + c2 * 64, tS + c2 * 64 + 32, sra, srb);
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const int c = 2 * c2 + hf;
                    uint32_t(&sr)[32] = hf ? srb : sra;
                    uint32_t pw[kPParts][8];
#pragma unroll
                    for (int g = 0; g < 8; ++g) {
                        float w4[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int key = k0 + c * 32 + 4 * g + u;
                            const float wv = ex2(__uint_as_float(sr[4 * g + u]) * row_factor - m16);
                            w4[u] = (full || key <= key_limit) ? wv : 0.f;
                            l4[u] += w4[u];
                        }
                        // Two keys at a time in f16x2 (11 bits, above the parts' 8): x = hi + lo + rest.
                        uint32_t hi = 0u, lo = 0u;
#pragma unroll
                        for (int pr = 0; pr < 2; ++pr) {
                            const __half2 x = __floats2half2_rn(w4[2 * pr], w4[2 * pr + 1]);
                            const uint32_t ch = __nv_cvt_halfraw2_to_fp8x2(__half2_raw(x), __NV_SATFINITE, __NV_E4M3);
                            const __half2 vh = __half2(__nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(ch), __NV_E4M3));
                            const uint32_t cl = __nv_cvt_halfraw2_to_fp8x2(__half2_raw(__hsub2(x, vh)), __NV_SATFINITE, __NV_E4M3);
                            const __half2 vl = __half2(__nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(cl), __NV_E4M3));
                            // What the PV product uses: the parts' sum (exact in f16).
                            const __half2 used = __hadd2(vh, vl);
                            lpv4[pr] = add_f16x2(lpv4[pr], *reinterpret_cast<const uint32_t *>(&used));
                            hi |= (ch & 0xffffu) << (16 * pr);
                            lo |= (cl & 0xffffu) << (16 * pr);
                        }
                        pw[0][g] = hi;
                        pw[1][g] = lo;
                    }
#pragma unroll
                    for (int pt = 0; pt < kPParts; ++pt)
                        tmem_st8(tS + 8u * kPParts * c + 8u * pt, pw[pt]);
                }
            }
            l += ((l4[0] + l4[1]) + (l4[2] + l4[3])) * (1.0f / kPScale);
            lpv += lpv4[0] + lpv4[1];
            tmem_wait_st();
            tc_fence_before_sync();
            mbar_arrive(BAR(kBarPFull));
        }
        // Epilogue: O * v_scale / lpv as bf16, LSE = (m_ref + log2(l)) ln 2, in natural-log units of
        // the scaled scores (l and m_ref are in units of the weights 2^(s - m_ref)).
        const bool okf = __all_sync(0xffffffffu, ok && mbar_wait(BAR(kBarODone), static_cast<uint32_t>(n_tiles - 1) & 1u,
                                                                 abort_flag, p.status, kSiteFp8Prefill));
        if (okf) {
            tc_fence_after_sync();
            const bool store = qi < p.Sq;
            const size_t row = (static_cast<size_t>(b) * p.Hq + h) * p.Sq + (store ? qi : 0);
            const float inv = lpv > 0.f ? 1.f / lpv : 0.f;
            const float *vs = p.v_scale + static_cast<size_t>(kvh) * kD;
            __nv_bfloat16 *orow = p.o + row * kD;
#pragma unroll 1
            for (int c = 0; c < kD / 32; ++c) {
                uint32_t ov[32];
                tmem_ld32_wait(tO + c * 32, ov);
                if (store) {
                    uint32_t pk[16];
#pragma unroll
                    for (int u = 0; u < 16; ++u) {
                        const float a = __uint_as_float(ov[2 * u]) * inv * vs[c * 32 + 2 * u];
                        const float bb = __uint_as_float(ov[2 * u + 1]) * inv * vs[c * 32 + 2 * u + 1];
                        __nv_bfloat162 v2 = __floats2bfloat162_rn(a, bb);
                        pk[u] = *reinterpret_cast<uint32_t *>(&v2);
                    }
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + c * 32);
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        dst[u] = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
                }
                __syncwarp();
            }
            if (store)
                p.lse[row] = (m_ref + log2f(l)) * 0.6931471805599453f;
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
#undef BAR
}

}  // namespace

cudaError_t launch_prefill_fp8(const PrefillFp8Args &a, cudaStream_t stream, int *encode_error)
{
    if (a.D != kD)
        return cudaErrorInvalidValue;
    static bool attr_set[kMaxDevices] = {};  // per device: the attribute applies to the current one
    const int dev = current_device_index();
    if (dev < 0)
        return cudaErrorInvalidDevice;
    if (!attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(prefill_fp8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
        if (e != cudaSuccess)
            return e;
        attr_set[dev] = true;
    }
    auto encode = get_encode_fn();
    if (!encode) {
        *encode_error = -1;
        return cudaErrorInitializationError;
    }
    CUtensorMap tk, tv;
    if (!make_map_u8(encode, &tk, a.k8, kD, a.Skv, a.B * a.Hkv, 128, kBN, CU_TENSOR_MAP_SWIZZLE_128B, encode_error) ||
        !make_map_u8(encode, &tv, a.v8, kD, a.Skv, a.B * a.Hkv, 128, kBN, CU_TENSOR_MAP_SWIZZLE_128B, encode_error))
        return cudaErrorInvalidValue;
    Fp8PrefillParams p;
    p.q = static_cast<const __nv_bfloat16 *>(a.q);
    p.k_scale = a.k_scale;
    p.v_scale = a.v_scale;
    p.o = static_cast<__nv_bfloat16 *>(a.o);
    p.lse = a.lse;
    p.status = a.status;
    p.B = a.B;
    p.Hq = a.Hq;
    p.Hkv = a.Hkv;
    p.Sq = a.Sq;
    p.Skv = a.Skv;
    p.group = a.Hq / a.Hkv;
    p.offset = a.Skv - a.Sq;
    p.causal = a.causal;
    p.n_qtiles = (a.Sq + kBM - 1) / kBM;
    p.scale_log2 = a.scale * kLog2e;
    const long long grid = static_cast<long long>(p.n_qtiles) * a.Hq * a.B;
    if (grid < 1 || grid > 0x7fffffffLL)
        return cudaErrorInvalidValue;
    prefill_fp8_kernel<<<static_cast<unsigned>(grid), kThreads, kSmem, stream>>>(tk, tv, p);
    return cudaGetLastError();
}

}  // namespace attn_b200
