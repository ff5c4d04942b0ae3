/*
 * prefill_sm100.cu — fused causal attention forward for Sq > 1 on sm_100a.
 *
 * One CTA computes one tile of 128 query rows of one (batch, query head). Per KV tile of 128 keys:
 *
 *   S = Q K^T          tcgen05.mma, bf16 operands in shared memory (TMA-loaded, 128B swizzle),
 *                      fp32 accumulator in tensor memory (TMEM), double-buffered so the next
 *                      tile's S is computed while this tile's softmax runs;
 *   online softmax     one query row per thread (TMEM lane = row): scale, cache-aligned causal
 *                      mask on diagonal tiles only, running max m and running sum l, rescale of the
 *                      O accumulator by exp(m_old - m_new);
 *   O += P V           P rounded to bf16 into shared memory, tcgen05.mma with V read MN-major
 *                      (O is divided by the sum of these rounded weights; the LSE uses the sum of
 *                      the exact fp32 weights);
 *   epilogue           O / l to bf16, LSE = (m + log2 l) * ln 2.
 *
 * Sources (page title, section): the fused single sweep over K/V per Q tile with S and P never
 * written to HBM — "AI Infra 入门：RMSNorm、Softmax、Causal Mask、Sampling 的数学与底层优化", §3
 * (FlashAttention paragraph); blocks above the diagonal skipped, blocks below computed unmasked,
 * only diagonal-crossing blocks masked — same page, §3 (block-sparse causal tiling); running max
 * and sum with the exp(m_old - m_new) rescale, which must also be applied to the output
 * accumulator — same page §3 and "Bộ 06 · Bên trong model", Q1; the mask aligned to the last Sq
 * key columns — "第11节：Attention 实现（Flash vs Fallback）", §3; bf16 storage with fp32
 * accumulation — "MLA 矩阵乘法吸收的数值稳定性治理", §二.2 and §五.
 *
 * Rescale threshold: the running max used for the exponentials is only moved when the new row
 * max exceeds it by more than 8 (in log2 units). The exponentials are then at most 2^8, which bf16
 * P and the fp32 sums hold without loss, and O and l stay consistent because both are accumulated
 * against the same reference max; the final O / l and LSE = m_ref + log2 l are the same quantities
 * as with an exact running max.
 *
 * Warp roles (192 threads): warps 0-3 softmax + correction + epilogue (warp w owns TMEM lanes
 * 32w..32w+31), warp 4 TMA producer, warp 5 TMEM allocator and MMA issuer (one thread issues).
 */
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <mutex>

#include "kernels.h"
#include "sm100_ptx.cuh"

namespace attn_b200 {
namespace {

constexpr int kBM = 128;  // query rows per tile = TMEM lanes = MMA M
constexpr int kBN = 128;  // keys per KV tile = MMA N of S and K of PV
constexpr int kRing = 4;  // K/V tile slots
constexpr int kSoftmaxWarps = 4;
constexpr int kWarpTma = 4;
constexpr int kWarpMma = 5;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;  // S0 [0,128), S1 [128,256), O [256, 256+D)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;

template <int D>
struct Cfg {
    static constexpr int kSwizzleBytes = (D * 2 >= 128) ? 128 : D * 2;  // 128 (D >= 64) or 64 (D = 32)
    static constexpr uint32_t kSwizzleMode = (kSwizzleBytes == 128) ? kSwizzle128B : kSwizzle64B;
    static constexpr int kChunkElems = kSwizzleBytes / 2;  // elements in one swizzled row
    static constexpr int kChunks = D / kChunkElems;
    static constexpr int kChunkBytes = 128 * kSwizzleBytes;  // 128 rows of one column block
    static constexpr int kTileBytes = 128 * D * 2;
    static constexpr int kPBytes = kBM * kBN * 2;
    static constexpr int kOffQ = 0;
    static constexpr int kOffRing = kOffQ + kTileBytes;
    static constexpr int kOffP = kOffRing + kRing * kTileBytes;
    static constexpr int kOffBar = kOffP + kPBytes;
    static constexpr int kUsed = kOffBar + 256;
    // >= 118 KB so that two CTAs never share an SM: each one allocates all 512 TMEM columns.
    static constexpr int kSmem = (kUsed + 1024 > 118 * 1024) ? kUsed + 1024 : 118 * 1024;
    static_assert(D % kChunkElems == 0, "head dim must be a whole number of swizzle rows");
    static_assert(kUsed + 1024 <= 227 * 1024, "shared memory budget");
};

enum Bar : int {
    kBarQ = 0,
    kBarFull0 = 1,
    kBarEmpty0 = kBarFull0 + kRing,
    kBarSFull0 = kBarEmpty0 + kRing,
    kBarSFree0 = kBarSFull0 + 2,
    kBarPFull = kBarSFree0 + 2,
    kBarODone = kBarPFull + 1,
    kBarDrain = kBarODone + 1,
    kNumBars = kBarDrain + 1,
};
static_assert(kNumBars * 8 <= 128, "barrier area");

struct Params {
    __nv_bfloat16 *o;
    float *lse;
    int *status;
    int B, Hq, Hkv, Sq, Skv, group, offset, causal, n_qtiles;
    float scale_log2;
};

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}

// Wait that ignores the abort flag (used to drain in-flight async work before exit).
__device__ __forceinline__ bool mbar_wait_drain(uint32_t bar, uint32_t parity, uint64_t limit_ns)
{
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > limit_ns)
            return false;
    }
    return true;
}

// Order in which K and V tiles are loaded and consumed: K0, K1, V0, K2, V1, ..., K(n-1), V(n-2), V(n-1).
__device__ __forceinline__ void kv_item(int it, int n_kv, int &tile, bool &is_v)
{
    if (it == 0) {
        tile = 0;
        is_v = false;
        return;
    }
    const int u = it - 1;
    const int j = u >> 1;
    if ((u & 1) == 0 && j + 1 < n_kv) {
        tile = j + 1;
        is_v = false;
    } else {
        tile = j;
        is_v = true;
    }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const Params p)
{
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t s_base = smem_u32(smem);
    const uint32_t sQ = s_base + C::kOffQ;
    const uint32_t sRing = s_base + C::kOffRing;
    const uint32_t sP = s_base + C::kOffP;
    const uint32_t bar0 = s_base + C::kOffBar;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kOffBar + 128);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::kOffBar + 132);
#define BAR(i) (bar0 + 8u * static_cast<uint32_t>(i))

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // Tile decode: heads fastest, then batch, then query tiles from the last (heaviest) one.
    int t = blockIdx.x;
    const int h = t % p.Hq;
    t /= p.Hq;
    const int b = t % p.B;
    t /= p.B;
    const int qt = p.n_qtiles - 1 - t;
    const int q0 = qt * kBM;
    const int bh_q = b * p.Hq + h;
    const int bh_kv = b * p.Hkv + h / p.group;

    // Keys visible to any row of this tile: [0, kv_end). Tiles past it are skipped entirely.
    int kv_end = p.Skv;
    if (p.causal)
        kv_end = min(p.Skv, q0 + kBM + p.offset);
    const int n_kv = (kv_end + kBN - 1) / kBN;

    if (threadIdx.x == 0) {
        mbar_init(BAR(kBarQ), 1);
        for (int r = 0; r < kRing; ++r) {
            mbar_init(BAR(kBarFull0 + r), 1);
            mbar_init(BAR(kBarEmpty0 + r), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(BAR(kBarSFull0 + i), 1);
            mbar_init(BAR(kBarSFree0 + i), kSoftmaxWarps * 32);
        }
        mbar_init(BAR(kBarPFull), kSoftmaxWarps * 32);
        mbar_init(BAR(kBarODone), 1);
        mbar_init(BAR(kBarDrain), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kWarpTma && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
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
            const uint64_t pol = l2_policy_evict_last();  // K/V tiles are re-read by sibling CTAs
            mbar_arrive_expect_tx(BAR(kBarQ), C::kTileBytes);
#pragma unroll
            for (int c = 0; c < C::kChunks; ++c)
                tma_load_3d(sQ + c * C::kChunkBytes, &tm_q, BAR(kBarQ), c * C::kChunkElems, q0, bh_q);
            const int n_items = 2 * n_kv;
            int issued = 0;
            for (int it = 0; it < n_items; ++it) {
                int tile;
                bool is_v;
                kv_item(it, n_kv, tile, is_v);
                const int slot = it % kRing;
                const uint32_t round = static_cast<uint32_t>(it / kRing);
                if (!mbar_wait(BAR(kBarEmpty0 + slot), (round & 1u) ^ 1u, abort_flag, p.status, kSitePrefillTmaEmpty))
                    break;
                mbar_arrive_expect_tx(BAR(kBarFull0 + slot), C::kTileBytes);
                const CUtensorMap *map = is_v ? &tm_v : &tm_k;
                const uint32_t dst = sRing + slot * C::kTileBytes;
#pragma unroll
                for (int c = 0; c < C::kChunks; ++c)
                    tma_load_3d_hint(dst + c * C::kChunkBytes, map, BAR(kBarFull0 + slot), c * C::kChunkElems,
                                     tile * kBN, bh_kv, pol);
                ++issued;
            }
            if (*abort_flag) {
                // Let every copy already issued land before the CTA exits.
                mbar_wait_drain(BAR(kBarQ), 0, 100000000ull);
                for (int it = (issued > kRing ? issued - kRing : 0); it < issued; ++it)
                    mbar_wait_drain(BAR(kBarFull0 + it % kRing), static_cast<uint32_t>(it / kRing) & 1u,
                                    100000000ull);
            }
        }
    } else if (warp == kWarpMma) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdS = idesc_bf16_f32(kBM, kBN, false);
            constexpr uint32_t kIdO = idesc_bf16_f32(kBM, D, true);
            constexpr uint32_t kSbo = 8 * C::kSwizzleBytes;  // 8 rows of one swizzled column block
            const uint32_t tS0 = tmem;
            const uint32_t tO = tmem + 2 * kBN;
            int it = 0;

            auto issue_s = [&](uint32_t d_tmem, uint32_t sK) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const int c = kk / (C::kChunkElems / 16);
                    const int w = kk % (C::kChunkElems / 16);
                    const uint32_t off = c * C::kChunkBytes + w * 32;
                    tc_mma_ss(d_tmem, smem_desc(sQ + off, 16, kSbo, C::kSwizzleMode),
                              smem_desc(sK + off, 16, kSbo, C::kSwizzleMode), kIdS, kk > 0 ? 1u : 0u);
                }
            };
            auto issue_pv = [&](uint32_t sV, bool accumulate) {
#pragma unroll
                for (int kk = 0; kk < kBN / 16; ++kk) {
                    const uint32_t a_addr = sP + (kk >> 2) * (kBM * 128) + (kk & 3) * 32;
                    const uint32_t b_addr = sV + kk * 16 * C::kSwizzleBytes;
                    tc_mma_ss(tO, smem_desc(a_addr, 16, 1024, kSwizzle128B),
                              smem_desc(b_addr, C::kChunkBytes, kSbo, C::kSwizzleMode), kIdO,
                              (accumulate || kk > 0) ? 1u : 0u);
                }
            };

            bool ok = mbar_wait(BAR(kBarQ), 0, abort_flag, p.status, kSitePrefillMmaQ);
            if (ok) {
                const int slot = it % kRing;
                ok = mbar_wait(BAR(kBarFull0 + slot), static_cast<uint32_t>(it / kRing) & 1u, abort_flag, p.status,
                               kSitePrefillMmaFull);
                if (ok) {
                    tc_fence_after_sync();
                    issue_s(tS0, sRing + slot * C::kTileBytes);
                    tc_commit(BAR(kBarSFull0));
                    tc_commit(BAR(kBarEmpty0 + slot));
                    ++it;
                }
            }
            for (int j = 0; ok && j < n_kv; ++j) {
                if (j + 1 < n_kv) {
                    const int sb = (j + 1) & 1;
                    const uint32_t use = static_cast<uint32_t>((j + 1) >> 1);
                    if (!(ok = mbar_wait(BAR(kBarSFree0 + sb), (use & 1u) ^ 1u, abort_flag, p.status,
                                         kSitePrefillMmaSFree)))
                        break;
                    const int slot = it % kRing;
                    if (!(ok = mbar_wait(BAR(kBarFull0 + slot), static_cast<uint32_t>(it / kRing) & 1u, abort_flag,
                                         p.status, kSitePrefillMmaFull)))
                        break;
                    tc_fence_after_sync();
                    issue_s(tS0 + sb * kBN, sRing + slot * C::kTileBytes);
                    tc_commit(BAR(kBarSFull0 + sb));
                    tc_commit(BAR(kBarEmpty0 + slot));
                    ++it;
                }
                if (!(ok = mbar_wait(BAR(kBarPFull), static_cast<uint32_t>(j) & 1u, abort_flag, p.status,
                                     kSitePrefillMmaPFull)))
                    break;
                const int slot = it % kRing;
                if (!(ok = mbar_wait(BAR(kBarFull0 + slot), static_cast<uint32_t>(it / kRing) & 1u, abort_flag,
                                     p.status, kSitePrefillMmaFull)))
                    break;
                tc_fence_after_sync();
                issue_pv(sRing + slot * C::kTileBytes, j > 0);
                tc_commit(BAR(kBarODone));
                tc_commit(BAR(kBarEmpty0 + slot));
                ++it;
            }
            // Every MMA issued above has completed once this barrier flips.
            tc_commit(BAR(kBarDrain));
            if (!mbar_wait_drain(BAR(kBarDrain), 0, kWaitLimitNs)) {
                *abort_flag = 1;
                atomicExch(p.status, kSitePrefillDrain);
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- softmax / correction / epilogue
        const int r = threadIdx.x;  // row within the tile == TMEM lane
        const int row = q0 + r;
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        const uint32_t tO = tmem + lane_base + 2 * kBN;
        const float sl2 = p.scale_log2;
        float m = -INFINITY;  // reference max, log2-scaled units
        float l = 0.f;        // running sum of the exact fp32 weights (gives the LSE)
        float l_pv = 0.f;     // running sum of the bf16-rounded weights the PV product uses (normalises O)
        bool ok = true;

        for (int j = 0; j < n_kv; ++j) {
            const int sb = j & 1;
            if (!(ok = mbar_wait(BAR(kBarSFull0 + sb), static_cast<uint32_t>(j >> 1) & 1u, abort_flag, p.status,
                                 kSitePrefillSoftmaxSFull)))
                break;
            tc_fence_after_sync();
            uint32_t s_raw[kBN];
            tmem_ld128_wait(tmem + lane_base + sb * kBN, s_raw);
            tc_fence_before_sync();
            mbar_arrive(BAR(kBarSFree0 + sb));

            float x[kBN];
#pragma unroll
            for (int c = 0; c < kBN; ++c)
                x[c] = __uint_as_float(s_raw[c]);

            const int k0 = j * kBN;
            const bool need_mask = (k0 + kBN > p.Skv) || (p.causal && k0 + kBN - 1 > q0 + p.offset);
            if (need_mask) {
                int limit = p.Skv - 1 - k0;  // last visible column of this tile for this row
                if (p.causal)
                    limit = min(limit, row + p.offset - k0);
#pragma unroll
                for (int c = 0; c < kBN; ++c)
                    if (c > limit)
                        x[c] = -INFINITY;
            }
            float mx = x[0];
#pragma unroll
            for (int c = 1; c < kBN; ++c)
                mx = fmaxf(mx, x[c]);
            const float mx2 = mx * sl2;  // scale > 0, so the max commutes with scaling

            float alpha = 1.f;
            bool rescale = false;
            if (j == 0) {
                m = mx2;  // key 0 is visible to every row, so this is finite
            } else {
                const float m_new = fmaxf(m, mx2);
                rescale = __any_sync(0xffffffffu, m_new > m + kRescaleThreshold);
                if (rescale) {
                    alpha = ex2(m - m_new);
                    m = m_new;
                }
            }
            const float neg_m = -m;
            float rowsum = 0.f, rowsum_pv = 0.f;
            uint32_t pk[kBN / 2];
#pragma unroll
            for (int c = 0; c < kBN / 2; ++c) {
                const float p0 = ex2(fmaf(x[2 * c], sl2, neg_m));
                const float p1 = ex2(fmaf(x[2 * c + 1], sl2, neg_m));
                pk[c] = pack_bf16x2(p0, p1);
                rowsum += p0 + p1;
                // The bf16-rounded weights that the PV product uses are summed as well, so that
                // O is divided by exactly the weight it was built from (a key that dominates a row
                // then contributes its V row without the rounding error of its weight).
                rowsum_pv += __uint_as_float(pk[c] << 16) + __uint_as_float(pk[c] & 0xffff0000u);
            }
            l = l * alpha + rowsum;
            l_pv = l_pv * alpha + rowsum_pv;

            if (j > 0) {
                // O and the P buffer belong to the previous PV product until it completes.
                if (!(ok = mbar_wait(BAR(kBarODone), static_cast<uint32_t>(j - 1) & 1u, abort_flag, p.status,
                                     kSitePrefillSoftmaxODone)))
                    break;
                tc_fence_after_sync();
                if (rescale) {
#pragma unroll 1
                    for (int cc = 0; cc < D / 32; ++cc) {
                        uint32_t ov[32];
                        tmem_ld32_wait(tO + cc * 32, ov);
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
                        tmem_st32_wait(tO + cc * 32, ov);
                    }
                }
            }
            // P row -> K-major 128B-swizzled tile: 16-byte unit u of row r lands at unit u ^ (r & 7).
#pragma unroll
            for (int u = 0; u < kBN / 8; ++u) {
                const int chunk = u >> 3;
                const int uu = u & 7;
                const uint32_t addr = sP + chunk * (kBM * 128) + r * 128 + ((uu ^ (r & 7)) << 4);
                st_shared_v4(addr, pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            mbar_arrive(BAR(kBarPFull));
        }

        if (ok)
            ok = mbar_wait(BAR(kBarODone), static_cast<uint32_t>(n_kv - 1) & 1u, abort_flag, p.status,
                           kSitePrefillEpilogue);
        if (ok) {
            tc_fence_after_sync();
            const float inv_l = 1.f / l_pv;
            const bool store = row < p.Sq;
            __nv_bfloat16 *orow = p.o + (static_cast<size_t>(bh_q) * p.Sq + (store ? row : 0)) * D;
#pragma unroll 1
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t ov[32];
                tmem_ld32_wait(tO + cc * 32, ov);
                uint32_t pkd[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    pkd[i] = pack_bf16x2(__uint_as_float(ov[2 * i]) * inv_l, __uint_as_float(ov[2 * i + 1]) * inv_l);
                if (store) {
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + cc * 32);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        dst[i] = make_uint4(pkd[4 * i], pkd[4 * i + 1], pkd[4 * i + 2], pkd[4 * i + 3]);
                }
            }
            if (store)
                p.lse[static_cast<size_t>(bh_q) * p.Sq + row] = (m + log2f(l)) * kLn2;
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

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult qres;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qres) == cudaSuccess &&
            qres == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// 3-D map over [BH][S][D] bf16 with a box of (inner, 128 rows, 1).
bool make_map(PFN_cuTensorMapEncodeTiled_v12000 encode, CUtensorMap *map, const void *base, int D, int S, int BH,
              int box_inner, CUtensorMapSwizzle swizzle, int *err)
{
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(S), static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(S) * D * 2};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(box_inner), 128u, 1u};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        *err = static_cast<int>(r);
        return false;
    }
    return true;
}

template <int D>
cudaError_t launch(const PrefillArgs &a, cudaStream_t stream, int *encode_error)
{
    using C = Cfg<D>;
    auto encode = get_encode_fn();
    if (!encode) {
        *encode_error = -1;
        return cudaErrorInitializationError;
    }
    const CUtensorMapSwizzle swz =
        (C::kSwizzleBytes == 128) ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    CUtensorMap tq, tk, tv;
    if (!make_map(encode, &tq, a.q, D, a.Sq, a.B * a.Hq, C::kChunkElems, swz, encode_error) ||
        !make_map(encode, &tk, a.k, D, a.Skv, a.B * a.Hkv, C::kChunkElems, swz, encode_error) ||
        !make_map(encode, &tv, a.v, D, a.Skv, a.B * a.Hkv, C::kChunkElems, swz, encode_error))
        return cudaErrorInvalidValue;

    static bool attr_set = false;  // benign race: every caller sets the same value
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(prefill_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
        if (e != cudaSuccess)
            return e;
        attr_set = true;
    }
    Params p;
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
    const long long grid = static_cast<long long>(p.n_qtiles) * a.B * a.Hq;
    prefill_kernel<D><<<static_cast<unsigned>(grid), kThreads, C::kSmem, stream>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const PrefillArgs &a, cudaStream_t stream, int *encode_error)
{
    *encode_error = 0;
    switch (a.D) {
    case 32:
        return launch<32>(a, stream, encode_error);
    case 64:
        return launch<64>(a, stream, encode_error);
    case 128:
        return launch<128>(a, stream, encode_error);
    default:
        return cudaErrorInvalidValue;
    }
}

}  // namespace attn_b200
