/*
 * bwd_sm100.cu — backward pass of the fused attention (head dim 128) on sm_100a: given dO, the
 * gradients dQ, dK, dV, with the softmax weights recomputed from the LSE saved by the forward.
 *
 * Per row i and visible key j (P_ij = exp(s_ij - lse_i), D_i = dO_i . O_i):
 *   dV_j += P_ij dO_i,   dS_ij = P_ij (dO_i . v_j - D_i),
 *   dQ_i += scale dS_ij k_j,   dK_j += scale dS_ij q_i.
 *
 * Kernels:
 *   bwd_pre_kernel   D_i = dO_i . O_i and lse_i in log2 units, per row, into the workspace (rows
 *                    padded to whole 128-row tiles per (batch, head)), and the row's fp32 dq
 *                    accumulator cleared (no separate memset);
 *   bwd_kernel       one CTA per (128-key tile of K and V, batch, kv head); it walks every query
 *                    head of the kv head's group and every 128-row query tile that sees any of its
 *                    keys. Per step (one query tile), with keys in TMEM lanes:
 *                      S^T  = K Q^T      and  dP^T = V dO^T     (tcgen05.mma, both operands TMA tiles)
 *                      P^T, dS^T         warps 0-15 (thread = key; warpgroup g takes query columns
 *                                        [32 g, 32 g + 32)) recompute the weights from the LSE,
 *                                        apply the causal mask, form dS, and write P^T and dS^T back
 *                                        into TMEM as bf16 and dS into shared memory, in two chunks
 *                                        of 16 columns;
 *                      dK  += dS^T Q     (A = dS^T from TMEM, B = Q read MN-major)
 *                      dV  += P^T dO     (A = P^T from TMEM, B = dO read MN-major); both start on
 *                                        every warp's first chunk while the second is computed
 *                      dQ   = dS K       (A = dS from shared memory, B = K read MN-major)
 *                    the same warps (thread = query row, warpgroup g: dQ dims [32 g, 32 g + 32))
 *                    then copy dQ x scale out of TMEM into the step's Q/dO stage (free once the
 *                    products are done), and warp 18 adds it into the fp32 workspace with TMA
 *                    reduce-adds while the next step runs; dK and dV stay in TMEM until the last
 *                    step. The asynchronous reduction takes the 64 KB of dQ per step off the chain
 *                    (written by the warps themselves, it took a third of the step: the SM's store
 *                    bandwidth to L2, not the reductions, bounded it).
 *                    When the key tiles are fewer than the SMs and the group splits evenly, each
 *                    key tile is a cluster of two CTAs that walk half of the query heads each; at
 *                    the end CTA 1 stages its partial dK, dV (fp32) in its shared memory and CTA 0
 *                    reads them through the cluster's distributed shared memory, adds them to its
 *                    own and stores the sums;
 *   bwd_dq_kernel    dQ (fp32 workspace) -> bf16.
 *
 * TMEM (512 columns): [0,128) S^T, then P^T (bf16: warpgroup g's queries in [32 g, 32 g + 16));
 * [128,256) dP^T, then dS^T (likewise from column 128), then dQ; [256,384) dV; [384,512) dK. The MMAs of one thread run in issue order, so dK's read of dS^T is done before dQ overwrites
 * those columns, and dV's read of P^T before the next S^T. The next step's S^T product needs only
 * that order; its dP^T product waits until dQ is out of TMEM, so S^T overlaps the dQ drain.
 *
 * Sources (page title, section): the backward pass recomputes the weights from the LSE the forward
 * saved instead of storing them — "AI Infra 入门：RMSNorm、Softmax、Causal Mask、Sampling 的数学与底层
 * 优化", §3 (LSE paragraph); the causal mask and its alignment to the last Sq keys — same page §3 and
 * "第11节：Attention 实现（Flash vs Fallback）", §3; bf16 operands with fp32 accumulation — "MLA 矩阵
 * 乘法吸收的数值稳定性治理", §二.2. The gradient formulas are the derivative of the forward definition.
 */
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <type_traits>

#include "kernels.h"
#include "sm100_ptx.cuh"
#include "tma_host.h"

namespace attn_b200 {
namespace {

constexpr int kD = 128;
constexpr int kBK = 128;  // keys per CTA tile (TMEM lanes of S^T, dP^T, dV, dK)
constexpr int kBQ = 128;  // query rows per step
constexpr int kSoftWarps = 16;     // four warpgroups: warp w serves TMEM lanes 32 (w % 4) .. + 31
constexpr int kGroupCols = 32;     // query columns (and dQ, dK, dV dims) per warpgroup
constexpr int kThreads = 640;
constexpr int kWarpTma = 16;
constexpr int kWarpMma = 17;
constexpr int kWarpRed = 18;  // issues the dQ reduce-adds
constexpr float kLog2e = 1.4426950408889634f;

constexpr int kHalf = 128 * 128;      // 128 rows x 64 dims (or 64 keys) of bf16, 128-byte swizzle
constexpr int kTile = 2 * kHalf;      // one 128 x 128 bf16 tile
constexpr int kOffK = 0;
constexpr int kOffV = kOffK + kTile;
constexpr int kOffStage = kOffV + kTile;  // two stages of Q_i, dO_i
constexpr int kStageBytes = 2 * kTile;
constexpr int kOffDS = kOffStage + 2 * kStageBytes;  // dS (queries x keys), A operand of dQ
constexpr int kDqBox = 128 * 128;                   // 128 rows x 32 fp32 of dQ, 128-byte swizzle
constexpr int kOffVec = kOffDS + kTile;              // two stages of [lse2 | D] (128 floats each)
constexpr int kVecBytes = 2 * kBQ * 4;
constexpr int kOffBar = kOffVec + 2 * kVecBytes;
enum BwdBar : int {
    kBarKV = 0,
    kBarStageFull0 = 1,   // [2]
    kBarStageEmpty0 = 3,  // [2]: the products are done with Q, dO, and the stage's dQ has been reduced
    kBarSD = 5,           // S^T and dP^T ready
    kBarP0 = 6,           // P^T, dS^T of each warp's first 32 query columns in TMEM (256 arrivals)
    kBarP1 = 7,           // ... of all 64, and dS in shared memory (256 arrivals)
    kBarDQ = 8,           // dQ ready
    kBarDQFree0 = 9,      // [2], by stage: dQ out of TMEM and staged in shared memory (256 arrivals)
    kBarFinal = 11,       // every MMA done
    kBarPeerReady = 12,   // cluster of two, CTA 0: CTA 1's partial dK (phase 0), dV (phase 1) staged (512 arrivals)
    kBarPeerDone = 13,    // CTA 1: CTA 0 has read the staged dK (512 arrivals)
    kNumBwdBars = 14,
};
constexpr int kOffMisc = kOffBar + kNumBwdBars * 8;
constexpr int kSmem = kOffMisc + 64;  // the dynamic window starts 1024-aligned (no static smem)
static_assert(kSmem <= 227 * 1024, "shared memory budget");
constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 384;

struct BwdParams {
    __nv_bfloat16 *dk, *dv;
    const float *vec;    // [2][B*Hq][Sq_pad]: lse2 then D
    int *status;
    int B, Hq, Hkv, Sq, Skv, Sq_pad, group, offset, causal, n_ktiles;
    int n_split;  // CTAs per key tile (1, or 2 as a cluster), each with group / n_split of the query heads
    float scale, scale_log2;
};

// ---- a 2-CTA cluster's exchange through distributed shared memory ----------------------------
__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// The address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t peer_addr(uint32_t addr, uint32_t rank)
{
    uint32_t out;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(addr), "r"(rank));
    return out;
}
__device__ __forceinline__ float4 ld_cluster_f4(uint32_t addr)
{
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr)
                 : "memory");
    return v;
}
// Arrival (release at cluster scope) on an mbarrier of the peer CTA, given its cluster address.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_bar)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
}
// Bounded wait (acquire at cluster scope: the peer's writes before its arrival are visible after).
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity, uint64_t limit_ns)
{
    const uint64_t t0 = global_timer_ns();
    while (true) {
        uint32_t done;
        asm volatile("{\n\t.reg .pred q;\n\tmbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 q, [%1], %2;\n\t"
                     "selp.u32 %0, 1, 0, q;\n\t}"
                     : "=r"(done)
                     : "r"(bar), "r"(parity)
                     : "memory");
        if (done)
            return true;
        if (global_timer_ns() - t0 > limit_ns)
            return false;
    }
}
// Every thread of both CTAs: the cluster barrier (release / acquire).
__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

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

__device__ __forceinline__ bool wait_drain(uint32_t bar, uint32_t parity, uint64_t limit_ns)
{
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > limit_ns)
            return false;
    }
    return true;
}

// First query tile whose rows see key k0 (causal: row q sees k0 iff k0 <= q + offset).
__device__ __forceinline__ int first_qtile(const BwdParams &p, int k0)
{
    if (!p.causal)
        return 0;
    const int q_min = k0 - p.offset;  // smallest row that sees key k0
    return q_min <= 0 ? 0 : q_min / kBQ;
}

// Half a warp per query row, two rows per warp and step (grid-stride, 64-bit row indices): each lane
// reads 16 bytes of O and of dO, D_i = dO_i . O_i is summed over the half-warp, and lse_i goes to
// log2 units; the same lanes clear the row's fp32 dq accumulator (512 bytes) that the main kernel
// adds into.
__global__ void __launch_bounds__(256) bwd_pre_kernel(const __nv_bfloat16 *o, const __nv_bfloat16 *dout,
                                                     const float *lse, float *vec, float *dq_acc, long long rows,
                                                     int Sq, int Sq_pad, size_t total_pad)
{
    const int lane = threadIdx.x & 31;
    const int hl = lane & 15;  // lane within the row's half-warp
    const long long n_pairs = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
    for (long long pr = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; 2 * pr < rows;
         pr += n_pairs) {
        const long long row = 2 * pr + (lane >> 4);
        const bool valid = row < rows;
        float d = 0.f;
        if (valid) {
            const uint4 a = reinterpret_cast<const uint4 *>(o + static_cast<size_t>(row) * kD)[hl];
            const uint4 b = reinterpret_cast<const uint4 *>(dout + static_cast<size_t>(row) * kD)[hl];
            const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int u = 0; u < 4; ++u)
                d += __uint_as_float(aw[u] << 16) * __uint_as_float(bw[u] << 16) +
                     __uint_as_float(aw[u] & 0xffff0000u) * __uint_as_float(bw[u] & 0xffff0000u);
            float4 *acc = reinterpret_cast<float4 *>(dq_acc + static_cast<size_t>(row) * kD) + 2 * hl;
            acc[0] = make_float4(0.f, 0.f, 0.f, 0.f);
            acc[1] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int off = 8; off > 0; off >>= 1)
            d += __shfl_xor_sync(0xffffffffu, d, off);
        if (valid && hl == 0) {
            const long long bh = row / Sq, i = row % Sq;
            const size_t idx = static_cast<size_t>(bh) * Sq_pad + static_cast<size_t>(i);
            vec[idx] = lse[row] * kLog2e;
            vec[total_pad + idx] = d;
        }
    }
}

// dQ (fp32 accumulator) -> bf16, two 16-byte loads in flight per thread and step.
__global__ void __launch_bounds__(256) bwd_dq_kernel(const float4 *acc, uint2 *dq, long long n4)
{
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    for (long long t = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; t < n4; t += 2 * stride) {
        const bool second = t + stride < n4;
        const float4 a = acc[t];
        const float4 c = second ? acc[t + stride] : make_float4(0.f, 0.f, 0.f, 0.f);
        dq[t] = make_uint2(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w));
        if (second)
            dq[t + stride] = make_uint2(pack_bf16x2(c.x, c.y), pack_bf16x2(c.z, c.w));
    }
}

__global__ void __launch_bounds__(kThreads, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
               const __grid_constant__ CUtensorMap tm_dq, const BwdParams p)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t s_base = smem_u32(smem);
    const uint32_t sK = s_base + kOffK, sV = s_base + kOffV, sStage = s_base + kOffStage, sDS = s_base + kOffDS;
    const uint32_t bar0 = s_base + kOffBar;
#define BAR(i) (bar0 + 8u * static_cast<uint32_t>(i))
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffMisc + 4);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // The swizzled tiles need the 1024-byte alignment the window starts with; refuse to run
    // otherwise (the status word tells the caller).
    if (s_base & 1023u) {
        if (threadIdx.x == 0)
            atomicExch(p.status, kSiteBwd);
        return;
    }

    // Work decode: the head split fastest (a cluster's two CTAs), then kv heads, then batch, then key
    // tiles from the first (the most rows see them).
    int t = blockIdx.x;
    const int sp = t % p.n_split;
    t /= p.n_split;
    const int g = t % p.Hkv;
    t /= p.Hkv;
    const int b = t % p.B;
    const int kt = t / p.B;
    const int k0 = kt * kBK;
    const int bh_kv = b * p.Hkv + g;
    const int n_qtiles = (p.Sq + kBQ - 1) / kBQ;
    const int qt0 = first_qtile(p, k0);
    const int steps_per_head = (qt0 < n_qtiles) ? n_qtiles - qt0 : 0;
    const int heads = p.group / p.n_split;  // query heads of this CTA
    const int n_steps = steps_per_head * heads;
    auto step_head = [&](int s) { return g * p.group + sp * heads + s / steps_per_head; };
    auto step_q0 = [&](int s) { return (qt0 + s % steps_per_head) * kBQ; };

    if (threadIdx.x == 0) {
        mbar_init(BAR(kBarKV), 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(BAR(kBarStageFull0 + s), 1);
            mbar_init(BAR(kBarStageEmpty0 + s), 2);  // the MMA commit and the reducer
            mbar_init(BAR(kBarDQFree0 + s), 32 * kSoftWarps);
        }
        mbar_init(BAR(kBarSD), 1);
        mbar_init(BAR(kBarP0), 32 * kSoftWarps);
        mbar_init(BAR(kBarP1), 32 * kSoftWarps);
        mbar_init(BAR(kBarDQ), 1);
        mbar_init(BAR(kBarFinal), 1);
        mbar_init(BAR(kBarPeerReady), 32 * kSoftWarps);
        mbar_init(BAR(kBarPeerDone), 32 * kSoftWarps);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (p.n_split > 1)
        cluster_sync();  // both CTAs' barriers are initialised before any remote arrival
    const uint32_t tmem = *tmem_slot;

    if (warp == kWarpTma) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0 && n_steps > 0) {
            mbar_arrive_expect_tx(BAR(kBarKV), 2 * kTile);
            for (int hf = 0; hf < 2; ++hf) {
                tma_load_3d(sK + hf * kHalf, &tm_k, BAR(kBarKV), hf * 64, k0, bh_kv);
                tma_load_3d(sV + hf * kHalf, &tm_v, BAR(kBarKV), hf * 64, k0, bh_kv);
            }
            int s = 0;
            for (; s < n_steps; ++s) {
                const int st = s & 1;
                if (!mbar_wait(BAR(kBarStageEmpty0 + st), (static_cast<uint32_t>(s >> 1) & 1u) ^ 1u, abort_flag, p.status,
                               kSiteBwd))
                    break;
                const int h = step_head(s), q0 = step_q0(s);
                const int bh_q = b * p.Hq + h;
                const uint32_t dst = sStage + st * kStageBytes;
                const size_t vec_off = static_cast<size_t>(bh_q) * p.Sq_pad + q0;
                const size_t total_pad = static_cast<size_t>(p.B) * p.Hq * p.Sq_pad;
                mbar_arrive_expect_tx(BAR(kBarStageFull0 + st), kStageBytes + kVecBytes);
                for (int hf = 0; hf < 2; ++hf) {
                    tma_load_3d(dst + hf * kHalf, &tm_q, BAR(kBarStageFull0 + st), hf * 64, q0, bh_q);
                    tma_load_3d(dst + kTile + hf * kHalf, &tm_do, BAR(kBarStageFull0 + st), hf * 64, q0, bh_q);
                }
                const uint32_t vdst = s_base + kOffVec + st * kVecBytes;
                bulk_load(vdst, p.vec + vec_off, kBQ * 4, BAR(kBarStageFull0 + st));
                bulk_load(vdst + kBQ * 4, p.vec + total_pad + vec_off, kBQ * 4, BAR(kBarStageFull0 + st));
            }
            if (*abort_flag) {
                wait_drain(BAR(kBarKV), 0, 100000000ull);
                for (int c = (s > 2 ? s - 2 : 0); c < s; ++c)
                    wait_drain(BAR(kBarStageFull0 + (c & 1)), static_cast<uint32_t>(c >> 1) & 1u, 100000000ull);
            }
        }
    } else if (warp == kWarpMma) {
        // ---------------------------------------------------------------- MMA issuer
        const bool leader = elect_one();
        constexpr uint32_t kIdSS = idesc_bf16_f32_ab(128, 128, false, false);  // S^T, dP^T
        constexpr uint32_t kIdTS = idesc_bf16_f32_ab(128, 128, false, true);   // dV, dK: B read MN-major
        constexpr uint32_t kIdQ = idesc_bf16_f32_ab(128, 128, false, true);    // dQ: A = dS, B = K read MN-major
        auto kmaj = [](uint32_t base, int kk) {  // K-major tile, K step kk (16 elements)
            return smem_desc(base + (kk >> 2) * kHalf + (kk & 3) * 32, 16, 1024, kSwizzle128B);
        };
        // Packed P^T / dS^T of queries [16 kk, 16 kk + 16): each warpgroup's bf16 pairs sit at the
        // start of its own 32 fp32 columns (see the softmax warps).
        auto pcol = [](int kk) { return static_cast<uint32_t>((kk >> 1) * kGroupCols + (kk & 1) * 8); };
        auto mnmaj = [](uint32_t base, int kk) {  // MN-major tile, K step kk (16 rows of 128 bytes)
            return smem_desc(base + kk * 16 * 128, kHalf, 1024, kSwizzle128B);
        };
        auto commit = [&](int bar) {
            if (leader)
                tc_commit(BAR(bar));
        };
        bool ok = n_steps > 0 && mbar_wait(BAR(kBarKV), 0, abort_flag, p.status, kSiteBwd);
        for (int s = 0; ok && s < n_steps; ++s) {
            const int st = s & 1;
            const uint32_t sQ = sStage + st * kStageBytes, sDO = sQ + kTile;
            if (!(ok = mbar_wait(BAR(kBarStageFull0 + st), static_cast<uint32_t>(s >> 1) & 1u, abort_flag, p.status,
                                 kSiteBwd)))
                break;
            tc_fence_after_sync();
            if (leader) {
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk)
                    tc_mma_ss(tmem + kColS, kmaj(sK, kk), kmaj(sQ, kk), kIdSS, kk > 0 ? 1u : 0u);
            }
            // dP^T goes where the previous step's dQ is: wait until that is out of TMEM (S^T above
            // runs meanwhile).
            if (s > 0 && !(ok = mbar_wait(BAR(kBarDQFree0 + ((s - 1) & 1)), static_cast<uint32_t>((s - 1) >> 1) & 1u,
                                          abort_flag, p.status, kSiteBwd)))
                break;
            tc_fence_after_sync();
            if (leader) {
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk)
                    tc_mma_ss(tmem + kColDP, kmaj(sV, kk), kmaj(sDO, kk), kIdSS, kk > 0 ? 1u : 0u);
            }
            commit(kBarSD);
            // dK and dV over the query columns each softmax warp has finished first (16-query steps
            // 0, 1, 4, 5), then over the rest once the softmax is done.
            for (int half = 0; half < 2; ++half) {
                if (!(ok = mbar_wait(BAR(kBarP0 + half), static_cast<uint32_t>(s) & 1u, abort_flag, p.status, kSiteBwd)))
                    break;
                tc_fence_after_sync();
                if (leader) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {  // dK += dS^T Q
                        const int kk = 2 * i + half;
                        tc_mma_ts(tmem + kColDK, tmem + kColDP + pcol(kk), mnmaj(sQ, kk), kIdTS, (s > 0 || kk > 0) ? 1u : 0u);
                    }
#pragma unroll
                    for (int i = 0; i < 4; ++i) {  // dV += P^T dO
                        const int kk = 2 * i + half;
                        tc_mma_ts(tmem + kColDV, tmem + kColS + pcol(kk), mnmaj(sDO, kk), kIdTS, (s > 0 || kk > 0) ? 1u : 0u);
                    }
                }
            }
            if (!ok)
                break;
            if (leader) {
#pragma unroll
                for (int kk = 0; kk < kBK / 16; ++kk)  // dQ = dS K (queries in TMEM lanes), over dS^T
                    tc_mma_ss(tmem + kColDP, kmaj(sDS, kk), mnmaj(sK, kk), kIdQ, kk > 0 ? 1u : 0u);
            }
            commit(kBarDQ);
            commit(kBarStageEmpty0 + st);
        }
        commit(kBarFinal);
        if (!wait_drain(BAR(kBarFinal), 0, kWaitLimitNs) && leader) {
            *abort_flag = 1;
            atomicExch(p.status, kSiteBwd);
        }
        __syncwarp();
    } else if (warp == kWarpRed) {
        // ---------------------------------------------------------------- dQ reducer
        // One barrier per stage: a step's staged dQ cannot be followed by the same stage's next
        // staging before this warp has reduced it (the stage is reloaded only after the arrival
        // below), so a wait never misses a phase.
        if (lane == 0 && n_steps > 0) {
            for (int s = 0; s < n_steps; ++s) {
                const int st = s & 1;
                if (!mbar_wait(BAR(kBarDQFree0 + st), static_cast<uint32_t>(s >> 1) & 1u, abort_flag, p.status, kSiteBwd))
                    break;
                const int h = step_head(s), q0 = step_q0(s);
                const uint32_t src = sStage + st * kStageBytes;
                for (int c = 0; c < 4; ++c)
                    tma_reduce_add_3d(&tm_dq, src + c * kDqBox, 32 * c, q0, b * p.Hq + h);
                bulk_commit_group();
                bulk_wait_group_read0();  // the producer may load the stage again
                mbar_arrive(BAR(kBarStageEmpty0 + st));
            }
            bulk_wait_group0();  // every reduction has been performed before the CTA exits
        }
    } else if (warp < kSoftWarps) {
        // ---------------------------------------------------------------- softmax and dQ warps
        // Warps w, w + 4, w + 8, w + 12 share TMEM lanes 32 (w % 4) .. + 31 and split the 128 columns
        // of a step: warpgroup g takes query columns [32 g, 32 g + 32) of S^T and dP^T (thread = key),
        // then dQ dims [32 g, 32 g + 32) (thread = query row). Each group packs its P^T and dS^T (bf16) in
        // place at the start of its own columns, so no group writes what another still reads.
        const int grp = warp >> 2;
        const int kr = threadIdx.x & 127;  // key (softmax) or query row (dQ) within the tile == TMEM lane
        const int key = k0 + kr;
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_base + kColS + kGroupCols * grp, tDP = tmem + lane_base + kColDP + kGroupCols * grp;
        const uint32_t tQ = tmem + lane_base + kColDP + kGroupCols * grp;
        bool ok = true;
        for (int s = 0; s < n_steps; ++s) {
            const int st = s & 1;
            // tcgen05.ld/st are warp-collective: the warp goes on or stops as one.
            if (!(ok = __all_sync(0xffffffffu, mbar_wait(BAR(kBarSD), static_cast<uint32_t>(s) & 1u, abort_flag,
                                                         p.status, kSiteBwd))))
                break;
            tc_fence_after_sync();
            const int h = step_head(s), q0 = step_q0(s);
            const float *lse2 = reinterpret_cast<const float *>(smem + kOffVec + st * kVecBytes);
            const float *dvec = lse2 + kBQ;
            // Columns of this step's query tile that this key may feed: visible and inside Sq.
            int last_q = min(kBQ, p.Sq - q0) - 1;  // last valid column
            int first_q = 0;
            if (p.causal)
                first_q = max(0, key - p.offset - q0);  // row q sees key iff key <= q + offset
            const bool key_ok = key < p.Skv;
            uint8_t *dsrow_base = smem + kOffDS + (kr >> 6) * kHalf;
            const int kk = kr & 63;
#pragma unroll 1
            for (int c = 0; c < 2; ++c) {
                const int cq = kGroupCols * grp + 16 * c;  // first query column of this chunk
                uint32_t sr[16], dr[16];
                tmem_ld16x2_wait(tS + c * 16, tDP + c * 16, sr, dr);
                uint32_t pk[8], dk[8];
                auto body = [&](auto masked) {
#pragma unroll
                    for (int i4 = 0; i4 < 16; i4 += 4) {
                        const float4 x = *reinterpret_cast<const float4 *>(lse2 + cq + i4);
                        const float4 y = *reinterpret_cast<const float4 *>(dvec + cq + i4);
                        const float nl[4] = {-x.x, -x.y, -x.z, -x.w};
                        const float dv[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
                        for (int i = i4; i < i4 + 4; i += 2) {
                            float pe[2], ds[2];
#pragma unroll
                            for (int u = 0; u < 2; ++u) {
                                const int q = cq + i + u;
                                const float w = ex2(fmaf(__uint_as_float(sr[i + u]), p.scale_log2, nl[i - i4 + u]));
                                const float g = w * (__uint_as_float(dr[i + u]) - dv[i - i4 + u]);
                                if constexpr (decltype(masked)::value) {
                                    const bool vis = key_ok && q >= first_q && q <= last_q;
                                    pe[u] = vis ? w : 0.f;
                                    ds[u] = vis ? g : 0.f;
                                } else {
                                    pe[u] = w;
                                    ds[u] = g;
                                }
                            }
                            pk[i >> 1] = pack_bf16x2(pe[0], pe[1]);
                            dk[i >> 1] = pack_bf16x2(ds[0], ds[1]);
#pragma unroll
                            for (int u = 0; u < 2; ++u) {
                                const int q = cq + i + u;
                                *reinterpret_cast<uint16_t *>(dsrow_base + q * 128 + ((((kk >> 3) ^ (q & 7)) << 4) | ((kk & 7) << 1))) =
                                    static_cast<uint16_t>(u ? (dk[i >> 1] >> 16) : (dk[i >> 1] & 0xffffu));
                            }
                        }
                    }
                };
                if (key_ok && first_q <= cq && cq + 15 <= last_q)
                    body(std::false_type{});
                else
                    body(std::true_type{});
                tmem_st8x2_wait(tS + c * 8, pk, tDP + c * 8, dk);
                if (c == 1)
                    fence_proxy_async_smem();  // dS, for the dQ product
                tc_fence_before_sync();
                mbar_arrive(BAR(kBarP0 + c));
            }

            // dQ of this step (thread = query row), scaled, added into the fp32 accumulator.
            if (!(ok = __all_sync(0xffffffffu, mbar_wait(BAR(kBarDQ), static_cast<uint32_t>(s) & 1u, abort_flag,
                                                         p.status, kSiteBwd))))
                break;
            tc_fence_after_sync();
            {
                // dQ x scale into this step's Q/dO stage, which the products have finished with (the
                // dQ commit covers every earlier product): four boxes of 128 rows x 32 fp32 in the
                // 128-byte swizzle; the reducer warp adds them into the fp32 accumulator by TMA while
                // the next step runs.
                uint8_t *stage = smem + kOffStage + st * kStageBytes;
                uint32_t v[32];
                tmem_ld32_wait(tQ, v);
                uint8_t *row = stage + grp * kDqBox + kr * 128;
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    *reinterpret_cast<float4 *>(row + ((u ^ (kr & 7)) << 4)) =
                        make_float4(__uint_as_float(v[4 * u]) * p.scale, __uint_as_float(v[4 * u + 1]) * p.scale,
                                    __uint_as_float(v[4 * u + 2]) * p.scale, __uint_as_float(v[4 * u + 3]) * p.scale);
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            mbar_arrive(BAR(kBarDQFree0 + st));
        }
        // Epilogue: dims [32 grp, 32 grp + 32) of dK (scaled) and dV of this key. The whole warp
        // loads (tcgen05.ld is warp-collective); only the stores of keys past Skv are skipped.
        const bool okf = __all_sync(0xffffffffu, ok && mbar_wait(BAR(kBarFinal), 0, abort_flag, p.status, kSiteBwd));
        const bool key_store = key < p.Skv;
        uint32_t kv[32], vv[32];
        if (okf) {
            tc_fence_after_sync();
            if (n_steps > 0) {
                tmem_ld32x2_wait(tmem + lane_base + kColDK + kGroupCols * grp, tmem + lane_base + kColDV + kGroupCols * grp,
                                 kv, vv);
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    kv[i] = vv[i] = 0u;
            }
        }
        bool store_ok = okf;
        if (p.n_split > 1) {
            // The cluster's CTA 1 stages its partial dK, then dV (fp32, [key][dim] with the 16-byte
            // unit index XOR key % 32, in the K/V tiles, which no product reads any more); CTA 0
            // adds them to its own and stores the sums. Waits are bounded; the cluster barrier at
            // the end keeps both CTAs' shared memory alive until every access is done.
            const uint32_t rank = cluster_rank();
            const uint32_t buf = s_base + kOffK;
            auto unit = [&](int c) { return static_cast<uint32_t>(kr * 512 + (((grp * 8 + c) ^ (kr & 31)) << 4)); };
            for (int round = 0; round < 2; ++round) {
                uint32_t(&val)[32] = round ? vv : kv;
                if (rank == 1) {
                    if (okf) {
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            *reinterpret_cast<uint4 *>(smem + kOffK + unit(c)) =
                                make_uint4(val[4 * c], val[4 * c + 1], val[4 * c + 2], val[4 * c + 3]);
                        mbar_arrive_remote(peer_addr(BAR(kBarPeerReady), 0));
                    }
                    if (round == 0 && okf && !mbar_wait_cluster(BAR(kBarPeerDone), 0, kWaitLimitNs))
                        atomicExch(p.status, kSiteBwd);
                } else {
                    store_ok = store_ok && mbar_wait_cluster(BAR(kBarPeerReady), static_cast<uint32_t>(round), kWaitLimitNs);
                    if (store_ok) {
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            const float4 x = ld_cluster_f4(peer_addr(buf + unit(c), 1));
                            val[4 * c] = __float_as_uint(__uint_as_float(val[4 * c]) + x.x);
                            val[4 * c + 1] = __float_as_uint(__uint_as_float(val[4 * c + 1]) + x.y);
                            val[4 * c + 2] = __float_as_uint(__uint_as_float(val[4 * c + 2]) + x.z);
                            val[4 * c + 3] = __float_as_uint(__uint_as_float(val[4 * c + 3]) + x.w);
                        }
                    } else if (okf) {
                        atomicExch(p.status, kSiteBwd);
                    }
                    if (round == 0)
                        mbar_arrive_remote(peer_addr(BAR(kBarPeerDone), 1));
                }
            }
            store_ok = store_ok && rank == 0;
        }
        if (store_ok) {
            const size_t row = static_cast<size_t>(bh_kv) * p.Skv + (key_store ? key : 0);
            __nv_bfloat16 *dk_row = p.dk + row * kD + kGroupCols * grp;
            __nv_bfloat16 *dv_row = p.dv + row * kD + kGroupCols * grp;
            if (key_store) {
                uint4 *dkk = reinterpret_cast<uint4 *>(dk_row);
                uint4 *dvv = reinterpret_cast<uint4 *>(dv_row);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    dkk[i] = make_uint4(pack_bf16x2(__uint_as_float(kv[8 * i]) * p.scale, __uint_as_float(kv[8 * i + 1]) * p.scale),
                                        pack_bf16x2(__uint_as_float(kv[8 * i + 2]) * p.scale, __uint_as_float(kv[8 * i + 3]) * p.scale),
                                        pack_bf16x2(__uint_as_float(kv[8 * i + 4]) * p.scale, __uint_as_float(kv[8 * i + 5]) * p.scale),
                                        pack_bf16x2(__uint_as_float(kv[8 * i + 6]) * p.scale, __uint_as_float(kv[8 * i + 7]) * p.scale));
                    dvv[i] = make_uint4(pack_bf16x2(__uint_as_float(vv[8 * i]), __uint_as_float(vv[8 * i + 1])),
                                        pack_bf16x2(__uint_as_float(vv[8 * i + 2]), __uint_as_float(vv[8 * i + 3])),
                                        pack_bf16x2(__uint_as_float(vv[8 * i + 4]), __uint_as_float(vv[8 * i + 5])),
                                        pack_bf16x2(__uint_as_float(vv[8 * i + 6]), __uint_as_float(vv[8 * i + 7])));
                }
            }
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (p.n_split > 1)
        cluster_sync();  // neither CTA leaves while the other may still touch its shared memory
    if (warp == kWarpMma) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, 512);
    }
#undef BAR
}

}  // namespace

size_t bwd_workspace_bytes(int B, int Hq, int Sq, int D)
{
    const size_t sq_pad = (static_cast<size_t>(Sq) + kBQ - 1) / kBQ * kBQ;
    return static_cast<size_t>(B) * Hq * Sq * D * sizeof(float) + 2 * static_cast<size_t>(B) * Hq * sq_pad * sizeof(float);
}

cudaError_t launch_bwd(const BwdArgs &a, cudaStream_t stream, int *encode_error)
{
    if (a.D != kD)
        return cudaErrorInvalidValue;
    static bool attr_set[kMaxDevices] = {};  // per device: the attribute applies to the current one
    const int dev = current_device_index();
    if (dev < 0)
        return cudaErrorInvalidDevice;
    if (!attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
        if (e != cudaSuccess)
            return e;
        attr_set[dev] = true;
    }
    auto encode = get_encode_fn();
    if (!encode) {
        *encode_error = -1;
        return cudaErrorInitializationError;
    }
    CUtensorMap tq, tk, tv, tdo, tdq;
    if (!make_map(encode, &tq, a.q, kD, a.Sq, a.B * a.Hq, 64, kBQ, CU_TENSOR_MAP_SWIZZLE_128B, encode_error) ||
        !make_map(encode, &tdo, a.dout, kD, a.Sq, a.B * a.Hq, 64, kBQ, CU_TENSOR_MAP_SWIZZLE_128B, encode_error) ||
        !make_map(encode, &tk, a.k, kD, a.Skv, a.B * a.Hkv, 64, kBK, CU_TENSOR_MAP_SWIZZLE_128B, encode_error) ||
        !make_map(encode, &tv, a.v, kD, a.Skv, a.B * a.Hkv, 64, kBK, CU_TENSOR_MAP_SWIZZLE_128B, encode_error))
        return cudaErrorInvalidValue;

    const int Sq_pad = (a.Sq + kBQ - 1) / kBQ * kBQ;
    const size_t rows = static_cast<size_t>(a.B) * a.Hq * a.Sq;
    float *dq_acc = static_cast<float *>(a.ws);
    float *vec = dq_acc + rows * kD;
    if (!make_map_f32(encode, &tdq, dq_acc, kD, a.Sq, a.B * a.Hq, 32, kBQ, CU_TENSOR_MAP_SWIZZLE_128B, encode_error))
        return cudaErrorInvalidValue;
    const size_t total_pad = static_cast<size_t>(a.B) * a.Hq * Sq_pad;
    const size_t pre_blocks = (rows + 15) / 16;  // eight warps of two rows per block, at most 64K blocks (grid-stride)
    bwd_pre_kernel<<<static_cast<unsigned>(pre_blocks < 65536 ? pre_blocks : 65536), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(a.o), static_cast<const __nv_bfloat16 *>(a.dout), a.lse, vec, dq_acc,
        static_cast<long long>(rows), a.Sq, Sq_pad, total_pad);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return e;

    BwdParams p;
    p.dk = static_cast<__nv_bfloat16 *>(a.dk);
    p.dv = static_cast<__nv_bfloat16 *>(a.dv);
    p.vec = vec;
    p.status = a.status;
    p.B = a.B;
    p.Hq = a.Hq;
    p.Hkv = a.Hkv;
    p.Sq = a.Sq;
    p.Skv = a.Skv;
    p.Sq_pad = Sq_pad;
    p.group = a.Hq / a.Hkv;
    p.offset = a.Skv - a.Sq;
    p.causal = a.causal;
    p.n_ktiles = (a.Skv + kBK - 1) / kBK;
    // A grid of fewer key tiles than SMs leaves SMs idle: then each key tile's query heads are split
    // over a cluster of two CTAs (when the group splits evenly). Larger grids keep one CTA per key
    // tile, where the split's second set-up and exchange cost more than the balance gains.
    const long long tiles = static_cast<long long>(p.n_ktiles) * a.B * a.Hkv;
    p.n_split = ((a.Hq / a.Hkv) % 2 == 0 && tiles < a.sm_count) ? 2 : 1;
    p.scale = a.scale;
    p.scale_log2 = a.scale * kLog2e;
    const long long grid = static_cast<long long>(p.n_ktiles) * a.B * a.Hkv * p.n_split;
    if (p.n_split > 1) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(grid));
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = kSmem;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if ((e = cudaLaunchKernelEx(&cfg, bwd_kernel, tq, tk, tv, tdo, tdq, p)) != cudaSuccess)
            return e;
    } else {
        bwd_kernel<<<static_cast<unsigned>(grid), kThreads, kSmem, stream>>>(tq, tk, tv, tdo, tdq, p);
    }
    if ((e = cudaGetLastError()) != cudaSuccess)
        return e;
    const long long n4 = static_cast<long long>(rows) * kD / 4;
    const long long dq_blocks = (n4 + 2 * 256 - 1) / (2 * 256);  // two float4 per thread, at most 64K blocks
    bwd_dq_kernel<<<static_cast<unsigned>(dq_blocks < 65536 ? dq_blocks : 65536), 256, 0, stream>>>(
        reinterpret_cast<const float4 *>(dq_acc), static_cast<uint2 *>(a.dq), n4);
    return cudaGetLastError();
}

}  // namespace attn_b200
