/*
 * prefill_sm100.cu — fused causal attention forward for Sq > 1 on sm_100a.
 *
 * One CTA computes two consecutive 128-row query tiles (A and B) of one (batch, query head). Both
 * tiles stream the same K/V tiles of 128 keys, so each K/V tile is brought into shared memory once
 * for 256 query rows. Per KV tile j and per query tile X in {A, B}:
 *
 *   S_X = Q_X K_j^T    tcgen05.mma, bf16 Q and K in shared memory (TMA-loaded, 128B swizzle),
 *                      fp32 accumulator in tensor memory (TMEM);
 *   online softmax     one query row per thread (TMEM lane = row): scale to log2 units, the
 *                      cache-aligned causal mask on diagonal tiles only, running max and sum, and
 *                      the exp(m_old - m_new) rescale of the O_X accumulator in TMEM;
 *   O_X += P_X V_j     P_X rounded to bf16 and written back into TMEM over the first half of
 *                      S_X's columns, then tcgen05.mma with A = P_X read from TMEM and B = V_j read
 *                      MN-major from shared memory;
 *   epilogue           O_X / l_X to bf16, LSE = (m + log2 l) * ln 2; for D = 128, O leaves through
 *                      TMA tensor stores from a staging box per warp, so the warps start the next
 *                      item without waiting for their stores to drain.
 *
 * The two tiles ping-pong: while the softmax warps of A work on S_A(j), the tensor core runs
 * S_B(j) and the PV product and next S of B, and the other way round. Because the MMAs of one
 * thread execute in issue order, the commit that announces S_X(j) also proves that PV_X(j-1) has
 * finished, so the softmax may rescale O_X right away, and S_X(j+1) — issued after PV_X(j) — never
 * overwrites P_X(j) before it has been read.
 *
 * Sources (page title, section): the fused single sweep over K/V per Q tile with S and P never
 * written to HBM — "AI Infra 入门：RMSNorm、Softmax、Causal Mask、Sampling 的数学与底层优化", §3
 * (FlashAttention paragraph); blocks above the diagonal skipped, blocks below computed unmasked,
 * only diagonal-crossing blocks masked — same page, §3 (block-sparse causal tiling); running max
 * and sum with the exp(m_old - m_new) rescale, which must also be applied to the output
 * accumulator — same page §3 and "Bộ 06 · Bên trong model", Q1; the mask aligned to the last Sq
 * key columns — "第11节：Attention 实现（Flash vs Fallback）", §3; bf16 storage with fp32
 * accumulation — "MLA 矩阵乘法吸收的数值稳定性治理", §二.2 and §五; the tcgen05/TMEM design space
 * (two query tiles, P kept on chip, softmax warps separate from the MMA issuer) — "AI Infra 入门",
 * §3 (FA4 paragraph), taken as prior art.
 *
 * Rescale threshold: the running max used for the exponentials is only moved when the new row
 * max exceeds it by more than 8 (in log2 units). The exponentials are then at most 2^8, which bf16
 * P and the fp32 sums hold without loss, and O and l stay consistent because both are accumulated
 * against the same reference max; the final O / l and LSE = m_ref + log2 l are the same quantities
 * as with an exact running max. O is divided by the sum of the bf16-rounded weights it was built
 * from; the LSE uses the sum of the exact fp32 weights.
 *
 * Warp roles (384 threads): warps 0-3 softmax / correction / epilogue of tile A, warps 4-7 the
 * same for tile B (warp w owns TMEM lanes 32(w%4)..+31), warp 8 TMA producer, warp 9 TMEM
 * allocator and MMA issuer (the whole warp walks the schedule, one elected lane issues), warps
 * 10-11 idle. setmaxnreg moves registers from the third warpgroup to the two softmax warpgroups.
 * P_X is handed to the tensor core in two halves: PV on the first 64 keys starts while the softmax
 * computes the second half.
 */
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <climits>
#include <cmath>
#include <mutex>

#include "kernels.h"
#include "sm100_ptx.cuh"
#include "tma_host.h"

namespace attn_b200 {
namespace {

constexpr int kBM = 128;  // query rows per tile = TMEM lanes = MMA M
constexpr int kBN = 128;  // keys per KV tile = MMA N of S and K of PV
constexpr int kRing = 4;  // K/V tile slots
constexpr int kWarpTma = 8;
constexpr int kWarpMma = 9;
constexpr int kThreads = 384;  // three warpgroups: softmax A, softmax B, producer + MMA (+ 2 spare warps)
// Register split: the block is launched with kLaunchRegs per thread (the host checks the compiled
// count before every first launch); the producer/MMA warpgroup gives registers back and the two
// softmax warpgroups take them, so the three shares add up to exactly the launch allocation.
constexpr int kLaunchRegs = 168;
constexpr int kRegsSoftmax = 200;
constexpr int kRegsOther = 104;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsOther == kThreads * kLaunchRegs, "register split");
constexpr uint32_t kTmemCols = 512;  // S_A [0,128), S_B [128,256), O_A [256,384), O_B [384,512)
__host__ __device__ constexpr uint32_t col_s(int x) { return static_cast<uint32_t>(x) * 128u; }        // S_X
__host__ __device__ constexpr uint32_t col_o(int x) { return 256u + static_cast<uint32_t>(x) * 128u; }  // O_X
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
    static constexpr int kOffQ = 0;  // Q_A, then Q_B
    static constexpr int kOffRing = kOffQ + 2 * kTileBytes;
    // D = 128: O leaves through TMA stores, each softmax warp staging its 32 rows x 64 dims (4 KB,
    // 128-byte swizzle) at a time.
    static constexpr bool kTmaStore = (D == 128);
    static constexpr int kWarpStageBytes = 32 * 128;
    static constexpr int kOffStage = kOffRing + kRing * kTileBytes;
    static constexpr int kOffBar = kOffStage + (kTmaStore ? 8 * kWarpStageBytes : 0);
    static constexpr int kUsed = kOffBar + 256;
    // >= 118 KB so that two CTAs never share an SM: each one allocates all 512 TMEM columns.
    static constexpr int kSmem = (kUsed + 1024 > 118 * 1024) ? kUsed + 1024 : 118 * 1024;
    static_assert(D % kChunkElems == 0, "head dim must be a whole number of swizzle rows");
    static_assert(kUsed + 1024 <= 227 * 1024, "shared memory budget");
};

enum Bar : int {
    kBarQFull = 0,
    kBarQFree = 1,  // the Q tiles may be replaced (every S product of the item has completed)
    kBarFull0 = 2,
    kBarEmpty0 = kBarFull0 + kRing,
    kBarSFull0 = kBarEmpty0 + kRing,  // [A, B]
    kBarPHalf0 = kBarSFull0 + 2,      // [A, B] first half of P_X stored
    kBarPFull0 = kBarPHalf0 + 2,      // [A, B] all of P_X stored
    kBarOFinal0 = kBarPFull0 + 2,     // [A, B]
    kBarDrain = kBarOFinal0 + 2,
    kNumBars = kBarDrain + 1,
};
static_assert(kNumBars * 8 <= 192, "barrier area");

struct Params {
    __nv_bfloat16 *o;
    long long o_sb, o_sh, o_ss;  // element strides of o (batch, head, row)
    float *lse;
    int *status;
    int B, Hq, Hkv, Sq, Skv, group, offset, causal;
    int n_items;      // work items along the query dimension (see the work decode)
    int n_work;       // work items in all: n_items * B * (Hq / heads per item)
    int pair_heads;   // 1: tiles A and B are the same query tile of two heads sharing a kv head
    float scale_log2;
    // Paged, variable-length cache (the kernel's kPaged variant): K and V are
    // [num_pages][Hkv][page_size][D], sequence b's keys are its first seq_lens[b] keys (clamped to
    // [0, cap]) in the pages block_table[b][0..pages_per_seq).
    const int *seq_lens = nullptr;
    const int *block_table = nullptr;
    int num_pages = 0, page_size = 0, pages_per_seq = 0, cap = 0;
    // Paged: 1 when the (batch, query-tile) pairs are few enough (<= kMaxSorted) to be put in order of
    // their KV-tile count at the start of the kernel (the lengths are known on the device only).
    int sorted = 0;
};

// The sorted order of (batch, query-tile) pairs (e = b + B * item) and their KV-tile counts.
constexpr int kMaxSorted = 64;
__shared__ uint16_t s_pair_order[kMaxSorted];
__shared__ int s_pair_tiles[kMaxSorted];

// Tiled bulk store of a shared-memory box into global memory (4-D map), tracked by the issuing
// thread's bulk async-group. Elements outside the tensor are not written.
__device__ __forceinline__ void tma_store_4d(const CUtensorMap *map, uint32_t src, int c0, int c1, int c2, int c3)
{
    asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
                 : "memory");
}

// Reference max of a row that has seen no key yet (paged variant): finite, so that the weights of
// masked scores are 2^(-inf) = 0 rather than NaN, and far below any real score.
constexpr float kNoKeyMax = -1e30f;

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Three-input maximum (one instruction on sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// acc + lo + hi for the two bf16 values packed in w, each added with fp32 accumulation (mixed-
// precision adds: no separate widening of the bf16 halves).
__device__ __forceinline__ float add_bf16x2(float acc, uint32_t w)
{
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\t"
        "add.rn.f32.bf16 %0, lo, %0;\n\tadd.rn.f32.bf16 %0, hi, %0;\n\t}"
        : "+f"(acc)
        : "r"(w));
    return acc;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
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

// Number of KV tiles a 128-row query tile starting at q0 needs over skv keys with the causal
// offset off (0 if the tile lies past Sq, or, paged, if none of its rows sees a key).
__device__ __forceinline__ int kv_tiles_for(const Params &p, int q0, int skv, int off)
{
    if (q0 >= p.Sq)
        return 0;
    int kv_end = skv;
    if (p.causal)
        kv_end = min(skv, q0 + kBM + off);  // last visible key of the tile's last row, + 1
    return kv_end > 0 ? (kv_end + kBN - 1) / kBN : 0;
}

// The r-th work item of this CTA, or -1. Persistent CTAs take the heaviest-first list in snake
// order (round r left to right when r is even, right to left when odd), which balances the
// decreasing item sizes over the CTAs as well as a dynamic queue would, with no shared counter.
__device__ __forceinline__ int work_index(const Params &p, int r)
{
    const int g = static_cast<int>(gridDim.x);
    const int c = static_cast<int>(blockIdx.x);
    const long long w = static_cast<long long>(r) * g + ((r & 1) ? (g - 1 - c) : c);
    return w < p.n_work ? static_cast<int>(w) : -1;
}

// One work item: two 128-row query tiles X = 0 (A), 1 (B) that stream the same K/V tiles.
struct Item {
    int q0[2];     // first query row of each tile
    int hq[2];     // query head of each tile
    int b, kvh;    // batch entry and kv head
    int skv, off;  // keys of the sequence, and the causal offset skv - Sq
    int n[2];      // KV tiles each tile needs (0: the tile lies past Sq or sees no key)
    __device__ __forceinline__ int n_max() const { return max(n[0], n[1]); }
};

// Work item w, heaviest first (query tiles from the last). With pair_heads (the GQA group is even),
// tiles A and B are the same 128 query rows of heads 2k and 2k+1, which share a kv head: both need
// the same number of KV tiles, so they ping-pong to the last one. Otherwise they are two
// consecutive query tiles of one head, and B needs one KV tile more than A.
template <bool kPaged>
__device__ __forceinline__ Item decode_item(const Params &p, int w)
{
    const int heads_per_item = p.pair_heads ? 2 : 1;
    const int hpu = p.Hq / heads_per_item;
    int t = w;
    const int hu = t % hpu;
    t /= hpu;
    int b, item;
    if (kPaged && p.sorted) {
        const int e = s_pair_order[t];
        b = e % p.B;
        item = e / p.B;
    } else {
        b = t % p.B;
        item = p.n_items - 1 - t / p.B;
    }
    const int h_a = hu * heads_per_item;
    Item it;
    it.q0[0] = p.pair_heads ? item * kBM : item * 2 * kBM;
    it.q0[1] = p.pair_heads ? it.q0[0] : it.q0[0] + kBM;
    it.hq[0] = h_a;
    it.hq[1] = h_a + (p.pair_heads ? 1 : 0);
    it.b = b;
    it.kvh = h_a / p.group;
    if constexpr (kPaged) {
        it.skv = min(max(__ldg(p.seq_lens + b), 0), p.cap);
        it.off = it.skv - p.Sq;
    } else {
        it.skv = p.Skv;
        it.off = p.offset;
    }
    it.n[0] = kv_tiles_for(p, it.q0[0], it.skv, it.off);
    it.n[1] = kv_tiles_for(p, it.q0[1], it.skv, it.off);
    return it;
}

// The first of this CTA's items from the r-th on that has a KV tile to stream, or -1. Without a
// paged cache every item has one; with it, an item whose rows see no key at all is written by the
// softmax warps alone (O = 0, LSE = -inf) and the producer and the MMA issuer skip it.
template <bool kPaged>
__device__ __forceinline__ int next_active(const Params &p, int r)
{
    for (;; ++r) {
        const int w = work_index(p, r);
        if (w < 0 || !kPaged || decode_item<kPaged>(p, w).n_max() > 0)
            return w < 0 ? -1 : r;
    }
}

template <int D, bool kPaged>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o, const Params p)
{
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t s_base = smem_u32(smem);
    const uint32_t sQ = s_base + C::kOffQ;
    const uint32_t sRing = s_base + C::kOffRing;
    const uint32_t bar0 = s_base + C::kOffBar;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kOffBar + 192);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::kOffBar + 196);
#define BAR(i) (bar0 + 8u * static_cast<uint32_t>(i))

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(BAR(kBarQFull), 1);
        mbar_init(BAR(kBarQFree), 1);
        for (int r = 0; r < kRing; ++r) {
            mbar_init(BAR(kBarFull0 + r), 1);
            mbar_init(BAR(kBarEmpty0 + r), 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(BAR(kBarSFull0 + x), 1);
            mbar_init(BAR(kBarPHalf0 + x), 128);
            mbar_init(BAR(kBarPFull0 + x), 128);
            mbar_init(BAR(kBarOFinal0 + x), 1);
        }
        mbar_init(BAR(kBarDrain), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (kPaged && p.sorted && warp == 10) {
        // Heaviest first by the pairs' real KV-tile counts (ties: lower e first), ranked by one warp.
        const int n = p.B * p.n_items;
        for (int e = lane; e < n; e += 32) {
            const int b = e % p.B, item = e / p.B;
            const int skv = min(max(__ldg(p.seq_lens + b), 0), p.cap), off = skv - p.Sq;
            const int q0a = p.pair_heads ? item * kBM : item * 2 * kBM;
            const int q0b = p.pair_heads ? q0a : q0a + kBM;
            s_pair_tiles[e] = max(kv_tiles_for(p, q0a, skv, off), kv_tiles_for(p, q0b, skv, off));
        }
        __syncwarp();
        for (int e = lane; e < n; e += 32) {
            const int c = s_pair_tiles[e];
            int rank = 0;
            for (int f = 0; f < n; ++f) {
                const int cf = s_pair_tiles[f];
                rank += (cf > c || (cf == c && f < e)) ? 1 : 0;
            }
            s_pair_order[rank] = static_cast<uint16_t>(e);
        }
    }
    if (warp == kWarpTma && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        if constexpr (C::kTmaStore)
            tma_prefetch_desc(&tm_o);
    }
    if (warp == kWarpMma) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp >= 8) {
      // Third warpgroup: gives registers back, then splits into the producer and the MMA issuer.
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsOther));
      if (warp == kWarpTma) {
        // ---------------------------------------------------------------- TMA producer
        // Per item: Q_A (and Q_B) once the previous item's last S products have read the Q tiles,
        // then K0, V0, K1, V1, ... through the ring, whose position runs on across items.
        if (lane == 0) {
            const uint64_t pol = l2_policy_evict_last();  // K/V tiles are re-read by sibling CTAs
            uint32_t kv = 0;   // K/V loads issued so far
            int q_issued = 0;  // Q loads issued so far (one per item with a KV tile)
            bool ok = true;
            int pg[8], ip[8];  // paged: page and first slot of each box of the current KV tile
            for (int k = next_active<kPaged>(p, 0); ok && k >= 0; k = next_active<kPaged>(p, k + 1)) {
                const Item it = decode_item<kPaged>(p, work_index(p, k));
                if (q_issued > 0 && !(ok = mbar_wait(BAR(kBarQFree), static_cast<uint32_t>(q_issued - 1) & 1u,
                                                     abort_flag, p.status, kSitePrefillTmaEmpty)))
                    break;
                const int n_q = (it.n[1] > 0) ? 2 : 1;
                mbar_arrive_expect_tx(BAR(kBarQFull), n_q * C::kTileBytes);
#pragma unroll
                for (int x = 0; x < 2; ++x)
                    if (x < n_q)
#pragma unroll
                        for (int c = 0; c < C::kChunks; ++c)
                            tma_load_4d(sQ + x * C::kTileBytes + c * C::kChunkBytes, &tm_q, BAR(kBarQFull),
                                        c * C::kChunkElems, it.q0[x], it.hq[x], it.b);
                ++q_issued;
                const int n_loads = 2 * it.n_max();  // K0, V0, K1, V1, ...
                for (int i = 0; i < n_loads; ++i, ++kv) {
                    const uint32_t slot = kv % kRing;
                    if (!(ok = mbar_wait(BAR(kBarEmpty0 + slot), ((kv / kRing) & 1u) ^ 1u, abort_flag, p.status,
                                         kSitePrefillTmaEmpty)))
                        break;
                    mbar_arrive_expect_tx(BAR(kBarFull0 + slot), C::kTileBytes);
                    const CUtensorMap *map = (i & 1) ? &tm_v : &tm_k;
                    const uint32_t dst = sRing + slot * C::kTileBytes;
                    if constexpr (kPaged) {
                        // The tile's keys come page by page, in boxes of min(page_size, 128) rows. A
                        // box past the sequence's length, or whose block-table entry lies outside
                        // [0, num_pages), reads the page beyond the last one: zeros.
                        const int rows = min(p.page_size, kBN);
                        const int n_box = kBN / rows;
                        if ((i & 1) == 0) {  // K: look the pages up; V reuses them
                            const int k0 = (i >> 1) * kBN;
#pragma unroll
                            for (int l = 0; l < 8; ++l) {
                                const int key = k0 + l * rows;
                                int page = p.num_pages;
                                if (l < n_box && key < it.skv) {
                                    page = __ldg(p.block_table + static_cast<size_t>(it.b) * p.pages_per_seq +
                                                 key / p.page_size);
                                    if (page < 0 || page >= p.num_pages)
                                        page = p.num_pages;
                                }
                                pg[l] = page;
                                ip[l] = key % p.page_size;
                            }
                        }
#pragma unroll
                        for (int l = 0; l < 8; ++l)
                            if (l < n_box)
#pragma unroll
                                for (int c = 0; c < C::kChunks; ++c)
                                    tma_load_4d_hint(dst + c * C::kChunkBytes + l * rows * C::kSwizzleBytes, map,
                                                     BAR(kBarFull0 + slot), c * C::kChunkElems, ip[l], it.kvh, pg[l],
                                                     pol);
                    } else {
#pragma unroll
                        for (int c = 0; c < C::kChunks; ++c)
                            tma_load_4d_hint(dst + c * C::kChunkBytes, map, BAR(kBarFull0 + slot), c * C::kChunkElems,
                                             (i >> 1) * kBN, it.kvh, it.b, pol);
                    }
                }
            }
            if (*abort_flag) {
                // Let every copy already issued land before the CTA exits.
                if (q_issued > 0)
                    mbar_wait_drain(BAR(kBarQFull), static_cast<uint32_t>(q_issued - 1) & 1u, 100000000ull);
                for (uint32_t i = (kv > kRing ? kv - kRing : 0); i < kv; ++i)
                    mbar_wait_drain(BAR(kBarFull0 + i % kRing), (i / kRing) & 1u, 100000000ull);
            }
        }
    } else if (warp == kWarpMma) {
        // ---------------------------------------------------------------- MMA issuer
        // The whole warp walks the schedule, so every descriptor and wait is warp-uniform; the
        // elected lane (the same one throughout) issues the MMAs and the commits that track them.
        {
            constexpr uint32_t kIdS = idesc_bf16_f32(kBM, kBN, false);
            constexpr uint32_t kIdO = idesc_bf16_f32(kBM, D, true);
            constexpr uint32_t kSbo = 8 * C::kSwizzleBytes;  // 8 rows of one swizzled column block
            const bool leader = elect_one();
            // Descriptors of the tile bases; a K step moves the start address, which is the low
            // field (address >> 4, 14 bits) of the descriptor: every address here is below 2^18.
            // The three descriptors share their high word (stride offset, version, swizzle); only the
            // low word (start address >> 4, leading-dimension offset) differs, and a K step or a
            // ring slot only adds to the start address.
            const uint64_t desc_q0 = smem_desc(sQ, 16, kSbo, C::kSwizzleMode);
            const uint32_t desc_hi = static_cast<uint32_t>(desc_q0 >> 32);
            const uint32_t q_lo = static_cast<uint32_t>(desc_q0);
            const uint32_t k_lo = static_cast<uint32_t>(smem_desc(sRing, 16, kSbo, C::kSwizzleMode));
            const uint32_t v_lo = static_cast<uint32_t>(smem_desc(sRing, C::kChunkBytes, kSbo, C::kSwizzleMode));
            constexpr uint32_t kSlotStep = static_cast<uint32_t>(C::kTileBytes >> 4);  // one tile, in descriptor units

            auto issue_s = [&](int x, uint32_t slot) {
                const uint32_t dq = q_lo + static_cast<uint32_t>(x) * kSlotStep;  // Q_B follows Q_A
                const uint32_t dk = k_lo + slot * kSlotStep;
                if (leader) {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const int c = kk / (C::kChunkElems / 16);
                        const int w = kk % (C::kChunkElems / 16);
                        const uint32_t off = static_cast<uint32_t>((c * C::kChunkBytes + w * 32) >> 4);
                        tc_mma_ss_lo(tmem + col_s(x), dq + off, dk + off, desc_hi, kIdS, kk > 0 ? 1u : 0u);
                    }
                }
            };
            // PV for the keys of one half of the tile: kk in [half * kBN / 32, (half + 1) * kBN / 32).
            auto issue_pv = [&](int x, uint32_t slot, bool accumulate, int half) {
                const uint32_t dv = v_lo + slot * kSlotStep;
                if (leader) {
#pragma unroll
                    for (int kk = half * (kBN / 32); kk < (half + 1) * (kBN / 32); ++kk) {
                        // P_X: 16 keys = 8 packed columns per step, in the first half of S_X's columns.
                        const uint32_t off = static_cast<uint32_t>((kk * 16 * C::kSwizzleBytes) >> 4);
                        tc_mma_ts_lo(tmem + col_o(x), tmem + col_s(x) + kk * 8, dv + off, desc_hi, kIdO,
                                     (accumulate || kk > 0) ? 1u : 0u);
                    }
                }
            };
            auto commit = [&](int bar) {
                if (leader)
                    tc_commit(BAR(bar));
            };
            auto wait_kv = [&](uint32_t i) -> bool {
                return mbar_wait(BAR(kBarFull0 + i % kRing), (i / kRing) & 1u, abort_flag, p.status,
                                 kSitePrefillMmaFull);
            };

            bool ok = true;
            int r_cur = next_active<kPaged>(p, 0);  // this CTA's item index (items with KV tiles only)
            Item it{};
            if (r_cur >= 0) {
                // The first item's S_X(0); every later item's are issued during the item before it.
                it = decode_item<kPaged>(p, work_index(p, r_cur));
                ok = mbar_wait(BAR(kBarQFull), 0, abort_flag, p.status, kSitePrefillMmaQ) && wait_kv(0);
                if (ok) {
                    tc_fence_after_sync();
                    for (int x = 0; x < 2; ++x)
                        if (it.n[x] > 0) {
                            issue_s(x, 0);
                            commit(kBarSFull0 + x);
                        }
                    commit(kBarEmpty0 + 0);
                }
            }
            uint32_t kv_base = 0;           // ring position of the current item's K0
            uint32_t p_cnt[2] = {0u, 0u};   // P_X tiles consumed so far (phase of PHalf_X / PFull_X)
            for (int k = 0; ok && r_cur >= 0; ++k) {  // k: Q loads consumed so far (phase of QFull)
                const int r_next = next_active<kPaged>(p, r_cur + 1);
                const int w_next = (r_next >= 0) ? work_index(p, r_next) : -1;
                const Item nx = (w_next >= 0) ? decode_item<kPaged>(p, w_next) : Item{};
                const uint32_t kv_next = kv_base + 2u * static_cast<uint32_t>(it.n_max());  // next item's K0
                // The Q tiles may be replaced once every S product of this item has been issued (and,
                // by the commit, completed): the last S_X is S_X(n_X - 1), issued at j = n_X - 2.
                int last_s_left = (it.n[0] >= 2 ? 1 : 0) + (it.n[1] >= 2 ? 1 : 0);
                bool q_free = false;
                // Tile X is done with this item once its last PV is issued: then the next item's
                // S_X(0) may overwrite S_X (in-order execution keeps it behind that PV).
                bool pending[2] = {it.n[0] == 0, it.n[1] == 0};
                int next_s_left = (w_next >= 0) ? (nx.n[0] > 0 ? 1 : 0) + (nx.n[1] > 0 ? 1 : 0) : 0;
                bool next_ready = false;  // next item's Q and K0 have landed
                auto try_commit_q_free = [&]() {
                    if (!q_free && last_s_left == 0) {
                        commit(kBarQFree);
                        q_free = true;
                    }
                };
                // Issue the next item's pending S_X(0) products. Non-blocking unless `block`: a Q or
                // K0 still in flight leaves them pending, so the current item's PVs are not held up.
                auto flush_next = [&](bool block) -> bool {
                    if (!q_free)
                        return true;
#pragma unroll
                    for (int y = 0; y < 2; ++y) {
                        if (!pending[y])
                            continue;
                        if (w_next < 0 || nx.n[y] == 0) {
                            pending[y] = false;
                            continue;
                        }
                        if (!next_ready) {
                            const uint32_t qpar = static_cast<uint32_t>(k + 1) & 1u;
                            const uint32_t kpar = (kv_next / kRing) & 1u;
                            const uint32_t kbar = BAR(kBarFull0 + kv_next % kRing);
                            if (block) {
                                if (!mbar_wait(BAR(kBarQFull), qpar, abort_flag, p.status, kSitePrefillMmaQ) ||
                                    !mbar_wait(kbar, kpar, abort_flag, p.status, kSitePrefillMmaFull))
                                    return false;
                            } else if (!__all_sync(0xffffffffu, mbar_try_wait(BAR(kBarQFull), qpar) &&
                                                                    mbar_try_wait(kbar, kpar))) {
                                return true;
                            }
                            next_ready = true;
                            tc_fence_after_sync();
                        }
                        issue_s(y, kv_next % kRing);
                        commit(kBarSFull0 + y);
                        pending[y] = false;
                        if (--next_s_left == 0)
                            commit(kBarEmpty0 + kv_next % kRing);  // both S products have read K0
                    }
                    return true;
                };
                try_commit_q_free();
                ok = flush_next(false);
                for (int j = 0; ok && j < it.n_max(); ++j) {
                    const uint32_t item_v = kv_base + 2u * j + 1u, item_k = kv_base + 2u * j + 2u;
                    if constexpr (kPaged) {
                        // Rows of V_j past the sequence's length hold whatever the cache holds in the
                        // last page's unused slots; their weights are 0, but 0 * NaN is not: zero them
                        // before the first PV product reads the tile.
                        const int r0 = it.skv - j * kBN;
                        if (r0 < kBN) {
                            if (!(ok = wait_kv(item_v)))
                                break;
                            uint4 *vt = reinterpret_cast<uint4 *>(smem + C::kOffRing + (item_v % kRing) * C::kTileBytes);
                            constexpr int kUnitsPerRow = C::kSwizzleBytes / 16;
                            for (int c = 0; c < C::kChunks; ++c)
                                for (int u = r0 * kUnitsPerRow + lane; u < kBN * kUnitsPerRow; u += 32)
                                    vt[c * (C::kChunkBytes / 16) + u] = make_uint4(0u, 0u, 0u, 0u);
                            fence_proxy_async_smem();
                            __syncwarp();
                        }
                    }
#pragma unroll
                    for (int x = 0; x < 2; ++x) {
                        if (!ok || j >= it.n[x])
                            continue;
                        // The first half of PV_X(j) runs while the softmax finishes the second half of P_X(j).
                        if (!(ok = mbar_wait(BAR(kBarPHalf0 + x), p_cnt[x] & 1u, abort_flag, p.status,
                                             kSitePrefillMmaPFull)))
                            continue;
                        if (!(ok = wait_kv(item_v)))
                            continue;
                        tc_fence_after_sync();
                        issue_pv(x, item_v % kRing, j > 0, 0);
                        if (!(ok = mbar_wait(BAR(kBarPFull0 + x), p_cnt[x] & 1u, abort_flag, p.status,
                                             kSitePrefillMmaPFull)))
                            continue;
                        ++p_cnt[x];
                        tc_fence_after_sync();
                        issue_pv(x, item_v % kRing, true, 1);
                        if (j + 1 < it.n[x]) {
                            if (!(ok = wait_kv(item_k)))
                                continue;
                            tc_fence_after_sync();
                            issue_s(x, item_k % kRing);
                            commit(kBarSFull0 + x);
                            if (j + 2 == it.n[x])
                                --last_s_left;
                        } else {
                            commit(kBarOFinal0 + x);
                            pending[x] = true;
                        }
                        try_commit_q_free();
                        ok = flush_next(false);
                    }
                    if (!ok)
                        break;
                    commit(kBarEmpty0 + item_v % kRing);
                    if (j + 1 < it.n_max())
                        commit(kBarEmpty0 + item_k % kRing);
                }
                if (ok)
                    ok = flush_next(true);
                kv_base = kv_next;
                it = nx;
                r_cur = r_next;
            }
            // Every MMA issued above has completed once this barrier flips.
            commit(kBarDrain);
            if (!mbar_wait_drain(BAR(kBarDrain), 0, kWaitLimitNs) && leader) {
                *abort_flag = 1;
                atomicExch(p.status, kSitePrefillDrain);
            }
        }
        __syncwarp();
      }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
        // ---------------------------------------------------------------- softmax / correction / epilogue
        const int x = warp >> 2;          // query tile: 0 = A, 1 = B
        const int r = threadIdx.x & 127;  // row within the tile == TMEM lane
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_base + col_s(x);
        const uint32_t tO = tmem + lane_base + col_o(x);
        const float sl2 = p.scale_log2;
        uint32_t phases = 0;  // bit 0: phase of SFull_X (one per S_X tile); bit 1: of OFinal_X (one per item)
        bool ok = true;

        // This tile's part of a work item. The next item's is decoded while the epilogue waits for
        // the last PV product (the integer divisions of a decode cost ~0.5 us of issue here), so the
        // next item's softmax starts right after the epilogue.
        struct Tile {
            int n = 0, q0 = 0, skv = 0, off = 0, hq = 0, b = 0;
        };
        auto tile_of = [&](int w) {
            const Item it = decode_item<kPaged>(p, w);
            Tile t;
            t.n = x ? it.n[1] : it.n[0];
            t.q0 = x ? it.q0[1] : it.q0[0];
            t.skv = it.skv;
            t.off = it.off;
            t.hq = x ? it.hq[1] : it.hq[0];
            t.b = it.b;
            return t;
        };
        int w = work_index(p, 0);
        Tile cur = (w >= 0) ? tile_of(w) : Tile{};
        Tile nxt{};
        int w_next = -1;
        for (int k = 0; ok && w >= 0; ++k, w = w_next, cur = nxt) {
            w_next = work_index(p, k + 1);
            const int n = cur.n, q0 = cur.q0, skv = cur.skv, off = cur.off;
            const int row = q0 + r;
            if (kPaged && n == 0 && q0 < p.Sq) {
                // Paged: a tile none of whose rows sees a key (the sequence holds fewer keys than
                // the rows before it): O = 0 and LSE = -inf, with no product to wait for.
                if (row < p.Sq) {
                    uint4 *dst = reinterpret_cast<uint4 *>(p.o + cur.b * p.o_sb + cur.hq * p.o_sh + row * p.o_ss);
#pragma unroll
                    for (int i = 0; i < D / 8; ++i)
                        dst[i] = make_uint4(0u, 0u, 0u, 0u);
                    p.lse[(static_cast<size_t>(cur.b) * p.Hq + cur.hq) * p.Sq + row] = -INFINITY;
                }
                nxt = (w_next >= 0) ? tile_of(w_next) : Tile{};
                continue;
            }
            float m = -INFINITY;  // reference max, log2-scaled units
            float l = 0.f;        // running sum of the exact fp32 weights (gives the LSE)
            float l_pv = 0.f;     // running sum of the bf16-rounded weights the PV product uses (normalises O)

            for (int j = 0; j < n; ++j) {
                // The wait's result gates the warp-collective TMEM load below: the warp agrees on it.
                if (!(ok = __all_sync(0xffffffffu, mbar_wait(BAR(kBarSFull0 + x), phases & 1u, abort_flag, p.status,
                                                             kSitePrefillSoftmaxSFull))))
                    break;
                phases ^= 1u;
                tc_fence_after_sync();
                uint32_t s_raw[kBN];
                tmem_ld128_wait(tS, s_raw);
                float s[kBN];
#pragma unroll
                for (int c = 0; c < kBN; ++c)
                    s[c] = __uint_as_float(s_raw[c]);

                const int k0 = j * kBN;
                const bool need_mask = (k0 + kBN > skv) || (p.causal && k0 + kBN - 1 > q0 + off);
                if (need_mask) {
                    int limit = skv - 1 - k0;  // last visible column of this tile for this row
                    if (p.causal)
                        limit = min(limit, row + off - k0);
#pragma unroll
                    for (int c = 0; c < kBN; ++c)
                        if (c > limit)
                            s[c] = -INFINITY;
                }
                // Row max: eight independent chains of three-input maxima.
                static_assert(kBN % 16 == 0, "row max walks the tile 16 columns at a time");
                float mx8[8];
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    mx8[i] = fmaxf(s[2 * i], s[2 * i + 1]);
#pragma unroll
                for (int c = 16; c < kBN; c += 16)
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        mx8[i] = fmax3(mx8[i], s[c + 2 * i], s[c + 2 * i + 1]);
                const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                                       fmaxf(mx8[6], mx8[7]));
                const float mx2 = mx * sl2;  // scale > 0, so the max commutes with scaling

                float alpha = 1.f;
                bool rescale = false;
                if (j == 0) {
                    // Key 0 is visible to every row, so this is finite; with a paged cache a row may
                    // see no key yet, and the floor keeps its weights 2^(-inf) = 0.
                    m = kPaged ? fmaxf(mx2, kNoKeyMax) : mx2;
                } else {
                    const float m_new = fmaxf(m, mx2);
                    rescale = __any_sync(0xffffffffu, m_new > m + kRescaleThreshold);
                    if (rescale) {
                        alpha = ex2(m - m_new);
                        m = m_new;
                    }
                }
                // O_X is stable here (the commit announcing S_X(j) came after PV_X(j-1)), and PV_X(j) is
                // not issued before the first arrival below, so the (rare) rescale fits in between.
                if (rescale) {
#pragma unroll 1
                    for (int cc = 0; cc < D / 32; ++cc) {
                        uint32_t ov[32];
                        tmem_ld32_wait(tO + cc * 32, ov);
#pragma unroll
                        for (int i = 0; i < 32; i += 2) {
                            const float2 v2 = __fmul2_rn(make_float2(__uint_as_float(ov[i]), __uint_as_float(ov[i + 1])),
                                                         make_float2(alpha, alpha));
                            ov[i] = __float_as_uint(v2.x);
                            ov[i + 1] = __float_as_uint(v2.y);
                        }
                        tmem_st32_wait(tO + cc * 32, ov);
                    }
                }
                // Exponentials, packed bf16 weights, and both running sums; P_X -> TMEM in two halves,
                // each announced as soon as it is stored so that the tensor core can start on it.
                const float2 sl2x2 = make_float2(sl2, sl2);
                const float2 negm2 = make_float2(-m, -m);
                float2 sum[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                                 make_float2(0.f, 0.f)};
                float sum_pv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t pk[32];
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const int col = half * 64 + 2 * c;
                        const float2 e = __ffma2_rn(make_float2(s[col], s[col + 1]), sl2x2, negm2);
                        const float2 pe = make_float2(ex2(e.x), ex2(e.y));
                        pk[c] = pack_bf16x2(pe.x, pe.y);
                        sum[c & 3] = __fadd2_rn(sum[c & 3], pe);
                        sum_pv[c & 3] = add_bf16x2(sum_pv[c & 3], pk[c]);
                    }
                    tmem_st32(tS + half * 32, pk);
                    tmem_wait_st();
                    tc_fence_before_sync();
                    mbar_arrive(BAR((half == 0 ? kBarPHalf0 : kBarPFull0) + x));
                }
                const float2 s01 = __fadd2_rn(__fadd2_rn(sum[0], sum[1]), __fadd2_rn(sum[2], sum[3]));
                const float q01 = (sum_pv[0] + sum_pv[1]) + (sum_pv[2] + sum_pv[3]);
                l = l * alpha + (s01.x + s01.y);
                l_pv = l_pv * alpha + q01;
            }
            nxt = (w_next >= 0) ? tile_of(w_next) : Tile{};
            if (!ok || n == 0)
                continue;

            // Epilogue. It overlaps the next item's first S product, which the issuer may start as
            // soon as PV_X(n-1) is issued; the next PV_X, which overwrites O_X, waits for this
            // warpgroup's first P arrival of the next item, which comes after these TMEM loads.
            ok = __all_sync(0xffffffffu, mbar_wait(BAR(kBarOFinal0 + x), (phases >> 1) & 1u, abort_flag, p.status,
                                                   kSitePrefillEpilogue));
            phases ^= 2u;
            if (!ok)
                break;
            tc_fence_after_sync();
            // Paged: a row that saw no key has l = 0: O = 0 and LSE = m + log2(0) = -inf.
            const float inv_l = (kPaged && !(l_pv > 0.f)) ? 0.f : 1.f / l_pv;
            const bool store = row < p.Sq;
            const int hq = cur.hq;
            const size_t bh_q = static_cast<size_t>(cur.b) * p.Hq + hq;
            if constexpr (C::kTmaStore) {
                // The warp's 32 rows, 64 dims at a time: TMEM -> bf16 -> the warp's staging box (rows of
                // 128 bytes, 16-byte units XOR row % 8: the 128-byte swizzle) -> one TMA store by lane 0.
                // The staging box is reused once the previous store has read it; rows past Sq are
                // clipped by the store.
                const uint32_t wstage = s_base + C::kOffStage + static_cast<uint32_t>(warp) * C::kWarpStageBytes;
                uint8_t *wrow = smem + C::kOffStage + warp * C::kWarpStageBytes + lane * 128;
                const int row0 = q0 + 32 * (warp & 3);
#pragma unroll 1
                for (int h = 0; h < D / 64; ++h) {
                    uint32_t oa[32], ob[32];
                    tmem_ld32x2_wait(tO + h * 64, tO + h * 64 + 32, oa, ob);
                    uint32_t pkd[32];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        pkd[i] = pack_bf16x2(__uint_as_float(oa[2 * i]) * inv_l, __uint_as_float(oa[2 * i + 1]) * inv_l);
                        pkd[16 + i] = pack_bf16x2(__uint_as_float(ob[2 * i]) * inv_l, __uint_as_float(ob[2 * i + 1]) * inv_l);
                    }
                    if (lane == 0)
                        bulk_wait_group_read0();
                    __syncwarp();
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        *reinterpret_cast<uint4 *>(wrow + ((u ^ (lane & 7)) << 4)) =
                            make_uint4(pkd[4 * u], pkd[4 * u + 1], pkd[4 * u + 2], pkd[4 * u + 3]);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0 && row0 < p.Sq) {
                        tma_store_4d(&tm_o, wstage, h * 64, row0, hq, cur.b);
                        bulk_commit_group();
                    }
                }
            } else {
                __nv_bfloat16 *orow = p.o + cur.b * p.o_sb + hq * p.o_sh + (store ? row : 0) * p.o_ss;
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
            }
            if (store)
                p.lse[bh_q * p.Sq + row] = (m + log2f(l)) * kLn2;
            tc_fence_before_sync();
        }
        if constexpr (C::kTmaStore) {
            // Every store issued by this warp has completed (its staging is read and O is written)
            // before the CTA can exit.
            if (lane == 0)
                bulk_wait_group0();
            __syncwarp();
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

template <int D, bool kPaged>
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
    CUtensorMap tq, tk, tv, to;
    auto st = [](const TensorStrides &t) { return Strides{t.b, t.h, t.s}; };
    if (!make_map4(encode, &tq, a.q, 2, D, a.Sq, a.Hq, a.B, st(a.qs), C::kChunkElems, 128, swz, encode_error))
        return cudaErrorInvalidValue;
    // O as (dim, row, head, batch), stored in boxes of 64 dims x 32 rows (one warp's rows); unused
    // (a copy of Q's map) without TMA stores.
    to = tq;
    if constexpr (C::kTmaStore)
        if (!make_map4(encode, &to, a.o, 2, D, a.Sq, a.Hq, a.B, st(a.os), 64, 32, CU_TENSOR_MAP_SWIZZLE_128B,
                       encode_error))
            return cudaErrorInvalidValue;
    if constexpr (kPaged) {
        // Pages [num_pages][Hkv][page_size][D] as (dim, slot, kv head, page), boxes of
        // min(page_size, 128) slots; the page index num_pages lies past the end: zeros.
        const Strides pst{static_cast<long long>(a.Hkv) * a.page_size * D, static_cast<long long>(a.page_size) * D, D};
        const int rows = a.page_size < kBN ? a.page_size : kBN;
        if (!make_map4(encode, &tk, a.k, 2, D, a.page_size, a.Hkv, a.num_pages, pst, C::kChunkElems, rows, swz,
                       encode_error) ||
            !make_map4(encode, &tv, a.v, 2, D, a.page_size, a.Hkv, a.num_pages, pst, C::kChunkElems, rows, swz,
                       encode_error))
            return cudaErrorInvalidValue;
    } else {
        if (!make_map4(encode, &tk, a.k, 2, D, a.Skv, a.Hkv, a.B, st(a.ks), C::kChunkElems, 128, swz, encode_error) ||
            !make_map4(encode, &tv, a.v, 2, D, a.Skv, a.Hkv, a.B, st(a.vs), C::kChunkElems, 128, swz, encode_error))
            return cudaErrorInvalidValue;
    }

    // Per device: the attribute applies to the device current when it is set (benign race between
    // host threads: every caller sets the same value).
    static bool attr_set[kMaxDevices] = {};
    const int dev = current_device_index();
    if (dev < 0)
        return cudaErrorInvalidDevice;
    if (!attr_set[dev]) {
        // The setmaxnreg split inside the kernel is only valid for the register count it was
        // written for; refuse to launch a build that was compiled to anything else.
        cudaFuncAttributes fa;
        cudaError_t e = cudaFuncGetAttributes(&fa, prefill_kernel<D, kPaged>);
        if (e != cudaSuccess)
            return e;
        if (fa.numRegs != kLaunchRegs)
            return cudaErrorInvalidConfiguration;
        e = cudaFuncSetAttribute(prefill_kernel<D, kPaged>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
        if (e != cudaSuccess)
            return e;
        attr_set[dev] = true;
    }
    Params p;
    p.o = static_cast<__nv_bfloat16 *>(a.o);
    p.o_sb = a.os.b;
    p.o_sh = a.os.h;
    p.o_ss = a.os.s;
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
    if constexpr (kPaged) {
        p.seq_lens = a.seq_lens;
        p.block_table = a.block_table;
        p.num_pages = a.num_pages;
        p.page_size = a.page_size;
        p.pages_per_seq = a.pages_per_seq;
        const long long cap = static_cast<long long>(a.pages_per_seq) * a.page_size;
        p.cap = static_cast<int>(cap < a.max_seq_len ? cap : a.max_seq_len);
    }
    const int n_qtiles = (a.Sq + kBM - 1) / kBM;
    p.pair_heads = (p.group % 2 == 0) ? 1 : 0;
    p.n_items = p.pair_heads ? n_qtiles : (n_qtiles + 1) / 2;
    p.sorted = (kPaged && static_cast<long long>(p.n_items) * a.B <= kMaxSorted) ? 1 : 0;
    p.scale_log2 = a.scale * kLog2e;
    const long long n_work = static_cast<long long>(p.n_items) * a.B * (a.Hq / (p.pair_heads ? 2 : 1));
    if (n_work > INT_MAX)
        return cudaErrorInvalidValue;
    p.n_work = static_cast<int>(n_work);
    // Persistent: one CTA per SM (each holds all 512 TMEM columns), never more than the items.
    const int grid = static_cast<int>(n_work < a.sm_count ? n_work : a.sm_count);
    prefill_kernel<D, kPaged><<<static_cast<unsigned>(grid), kThreads, C::kSmem, stream>>>(tq, tk, tv, to, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const PrefillArgs &a, cudaStream_t stream, int *encode_error)
{
    *encode_error = 0;
    if (a.seq_lens)  // paged, variable-length cache: head dim 128
        return a.D == 128 ? launch<128, true>(a, stream, encode_error) : cudaErrorInvalidValue;
    switch (a.D) {
    case 32:
        return launch<32, false>(a, stream, encode_error);
    case 64:
        return launch<64, false>(a, stream, encode_error);
    case 128:
        return launch<128, false>(a, stream, encode_error);
    default:
        return cudaErrorInvalidValue;
    }
}

}  // namespace attn_b200
