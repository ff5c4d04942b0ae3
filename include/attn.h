/*
 * attn.h — C ABI of libattn_b200.so: fused causal scaled-dot-product attention on B200 (sm_100a).
 *
 * The operation (per batch b, query head h, query row i; kv head = h / (Hq / Hkv)):
 *
 *   key j is visible to query i  iff  j < Skv  and  (!causal or j <= i + (Skv - Sq))
 *   s_j    = scale * (q_i . k_j)
 *   o_i    = sum_j softmax(s)_j * v_j          over the visible keys
 *   lse_i  = ln( sum_j exp(s_j) )              over the visible keys (natural log, scaled scores)
 *
 * Sources (page title, section):
 *   scores and the 1/sqrt(d) scale ... "05 · Tích vô hướng, Softmax và toán của Attention", §1 and
 *                                      "Vì sao chia cho √128";
 *   safe / online softmax, LSE ....... "AI Infra 入门：RMSNorm、Softmax、Causal Mask、Sampling 的数学与
 *                                      底层优化", §2-§3 (running max and sum rescaled by
 *                                      exp(m_old - m_new); LSE compresses (m, l) into one scalar and
 *                                      is the merge key of split-KV decoding);
 *   mask aligned to the last Sq keys . "第11节：Attention 实现（Flash vs Fallback）", §3 (the -inf upper
 *                                      triangle is added to the last seq_len key columns of a KV cache);
 *   decode needs no mask ............. "AI Infra 入门…", §3 (a single new query sees every cached key);
 *   grouped K/V heads ................ "05 · Tích vô hướng…", §4 (32 query heads share 8 K/V heads).
 *
 * Layout (all contiguous, row-major): q [B, Hq, Sq, D], k and v [B, Hkv, Skv, D], o [B, Hq, Sq, D],
 * all bf16; lse [B, Hq, Sq] fp32.
 *
 * Ownership: every pointer is a DEVICE pointer owned by the caller. The library keeps no pointer
 * after the work completes on `stream`. The library owns one small per-device workspace (the
 * split-KV partials of the decode kernel and a status word; attn_bwd keeps a second one). It grows
 * on the first call that needs more, stream-ordered: the new block is taken from the device's
 * stream-ordered pool on `stream` (cudaMallocAsync) and the old one released on `stream` after the
 * work queued before it (cudaFreeAsync); the host never waits. Make one call of the largest size
 * before capturing a stream into a CUDA graph. Calls on different streams of one device share the
 * workspace and must be serialised by the caller (an event between the streams suffices).
 *
 * Errors: argument errors are detected on the host before any launch and returned as a negative
 * attn_status; nothing is launched then. Launch failures return ATTN_ERR_LAUNCH. No call other
 * than attn_device_status synchronises; none aborts the process or traps on the device.
 * Kernel-side waits are bounded: a wait that runs out sets a device status word, which
 * attn_device_status() reads.
 */
#ifndef ATTN_B200_ATTN_H
#define ATTN_B200_ATTN_H

#ifdef __cplusplus
extern "C" {
#endif

typedef enum attn_status {
    ATTN_OK = 0,
    ATTN_ERR_NULL = -1,             /* a required pointer is NULL */
    ATTN_ERR_SHAPE = -2,            /* a size is < 1 or the problem exceeds the supported index range */
    ATTN_ERR_GQA = -3,              /* Hq is not a multiple of Hkv */
    ATTN_ERR_HEADDIM = -4,          /* D is not 32, 64 or 128 */
    ATTN_ERR_ALIGN = -5,            /* a pointer is not 16-byte aligned */
    ATTN_ERR_CAUSAL_SQ_GT_SKV = -6, /* causal with Sq > Skv: early rows would see no key */
    ATTN_ERR_ARCH = -7,             /* the current device is not compute capability 10.0 (sm_100a) */
    ATTN_ERR_WORKSPACE = -8,        /* the library workspace could not be allocated */
    ATTN_ERR_LAUNCH = -9,           /* a kernel launch failed */
    ATTN_ERR_DEVICE_TIMEOUT = -10,  /* a kernel-side wait ran out (reported by attn_device_status) */
    ATTN_ERR_SCALE = -11,           /* scale is not finite and > 0 */
    ATTN_ERR_CUDA = -12,            /* a CUDA runtime call failed (device query, tensor map, copy) */
    ATTN_ERR_SCRATCH_LIMIT = -13    /* attn_decode_noalloc: the problem needs more scratch than its fixed buffer */
} attn_status;

/*
 * attn_fwd — the whole forward pass: o and lse for every (b, h, i).
 *   q, k, v   device pointers, bf16, layouts above, 16-byte aligned.
 *   o         device pointer, bf16 [B, Hq, Sq, D], written entirely.
 *   lse       device pointer, fp32 [B, Hq, Sq], written entirely.
 *   B, Hq, Hkv, Sq, Skv, D   sizes; Hq % Hkv == 0; D in {32, 64, 128}.
 *   scale     multiplies q . k (normally 1/sqrt(D)); must be finite and > 0.
 *   causal    0 or 1. With Sq == 1 the mask hides nothing and both values give the same result.
 *   stream    a cudaStream_t (NULL = the legacy default stream).
 * Sq == 1 runs the split-KV decode kernel; every other shape runs the prefill kernel.
 * Returns ATTN_OK or a negative attn_status.
 */
int attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
             int B, int Hq, int Hkv, int Sq, int Skv, int D,
             float scale, int causal, void *stream);

/*
 * attn_fwd_ex — attn_fwd with the number of CTAs of the decode kernel fixed by the caller
 * (decode_ctas >= 1), or chosen by the library (decode_ctas == 0: one CTA per slot the GPU can keep
 * resident). The decode spreads the chunks of every (batch, kv head) key range evenly over those
 * CTAs, so this is a performance parameter: results agree with attn_fwd within rounding. Ignored
 * when Sq > 1.
 */
int attn_fwd_ex(const void *q, const void *k, const void *v, void *o, float *lse,
                int B, int Hq, int Hkv, int Sq, int Skv, int D,
                float scale, int causal, int decode_ctas, void *stream);

/*
 * attn_fwd_host — attn_fwd from host memory to host memory, with the copies pipelined against the
 * attention: the (batch, kv head) units are cut into up to ten slices, and while slice i is
 * copied in, slice i-1 is computed and slice i-2 is copied out (two copy streams of the library's
 * own, ordered against `stream` with events). When the group splits evenly (and half a group of
 * rows is a whole number of 16-byte blocks of lse), the first and the last unit go in two halves
 * of their query heads, which shortens the unoverlapped first copy in and last copy out. Same operation and results as attn_fwd on the same
 * values (each unit is computed the same way; the decode's split over CTAs may differ, within
 * rounding) — "第11节：Attention 实现（Flash vs Fallback）", §3 for the mask, as attn_fwd.
 *   q_host, k_host, v_host   host pointers, bf16, the contiguous layouts above. Page-locked
 *                            (pinned) memory lets the copies overlap the kernels; pageable memory
 *                            works but the copies then do not overlap.
 *   o_host, lse_host         host pointers, bf16 [B, Hq, Sq, D] and fp32 [B, Hq, Sq].
 *   q_dev .. lse_dev         device staging buffers of the same shapes, 16-byte aligned, owned by
 *                            the caller and not used by other work until the call's work is done.
 *   other arguments          as attn_fwd.
 * Ordering: the copies start after the work already queued on `stream`, and work queued on
 * `stream` after the call starts after the last copy back. The call returns once everything is
 * queued: synchronise `stream` before reading o_host and lse_host, and keep every buffer alive
 * until then. The first call on a device creates two streams and four events that live for the
 * process; otherwise the call allocates only what attn_fwd does. Calls from several host threads
 * queue one after another (they share those streams and events).
 * Returns ATTN_OK or a negative attn_status: ATTN_ERR_NULL for a null host or device pointer, the
 * attn_fwd errors for the shapes and the device buffers, ATTN_ERR_CUDA when a copy cannot be
 * queued (the streams are joined back into `stream` on every path).
 */
int attn_fwd_host(const void *q_host, const void *k_host, const void *v_host, void *o_host, float *lse_host,
                  void *q_dev, void *k_dev, void *v_dev, void *o_dev, float *lse_dev,
                  int B, int Hq, int Hkv, int Sq, int Skv, int D, float scale, int causal, void *stream);

/*
 * attn_fwd_strided — attn_fwd over tensors in any layout whose head dim is contiguous, e.g. the
 * token-major [B, S, H, D] that a projection writes, as well as the heads-major [B, H, S, D].
 *
 * Source (page title, section): the operation is attn_fwd's; the layout [B, H, Q_len, K_len] of the
 * scores in "第11节：Attention 实现（Flash vs Fallback）", §4 fixes no memory layout for q, k, v and o,
 * which is the caller's.
 *
 *   q_strides, k_strides, v_strides, o_strides   host arrays of three element strides each:
 *       {batch, head, row} — element (b, h, i, d) of q is q[b*s[0] + h*s[1] + i*s[2] + d]. Every
 *       stride must be >= 1, a multiple of 8 elements (16 bytes) and below 2^38; o's strides must
 *       not make two output elements share an address (not checked).
 *   lse       fp32 [B, Hq, Sq], contiguous, as for attn_fwd.
 * Every other argument, rule and return value is attn_fwd's; a stride triple that breaks the rule
 * above returns ATTN_ERR_ALIGN and NULL stride arrays ATTN_ERR_NULL, before any launch. A decode
 * (Sq == 1) with D = 32 or 64 in a layout other than the contiguous one runs the prefill kernel (the
 * CUDA-core decode kernel streams contiguous K/V rows only): correct, slower than attn_fwd's decode.
 */
int attn_fwd_strided(const void *q, const void *k, const void *v, void *o, float *lse,
                     int B, int Hq, int Hkv, int Sq, int Skv, int D,
                     const long long *q_strides, const long long *k_strides, const long long *v_strides,
                     const long long *o_strides, float scale, int causal, void *stream);

/* attn_decode_ctas — the number of CTAs attn_fwd would launch for a decode of this shape on the
 * current device (>= 1), or a negative attn_status. */
int attn_decode_ctas(int B, int Hq, int Hkv, int Skv, int D);

/* attn_status_string — a static, human-readable description of a status code. Never NULL. */
const char *attn_status_string(int status);

/* attn_version — library version as major * 10000 + minor * 100 + patch. */
int attn_version(void);

/*
 * attn_device_status — synchronises `stream`, then reads and clears the current device's status
 * words: the workspace's (every entry point except attn_decode_noalloc) and, once
 * attn_decode_noalloc has run on the device, the one in its fixed array. Returns ATTN_OK if no
 * kernel-side wait has run out since the last call,
 * ATTN_ERR_DEVICE_TIMEOUT if one has, or ATTN_ERR_CUDA if the stream could not be synchronised.
 * This is a diagnostic call: it blocks the host, so it does not belong on a hot path.
 */
int attn_device_status(void *stream);

/*
 * attn_decode_noalloc — single-token decode (Sq == 1) that allocates no memory.
 *
 * The pages have no counterpart to this entry point: it is an interface addition for callers that
 * must not have a library allocate device memory — a serving loop that cannot absorb the latency
 * of an allocation in the middle of a request, or a process whose device memory is owned by one
 * allocator or a budget fixed at start-up, where an allocation behind that allocator's back fails
 * or breaks its accounting. attn_fwd grows a workspace (cudaMallocAsync) on first use; this call
 * instead uses a fixed array of ATTN_DECODE_NOALLOC_SCRATCH_BYTES in the library's own device
 * memory, held on every GPU where it has been placed until the process exits. It calls no
 * cudaMalloc, cudaFree or other allocating routine.
 *
 * Arguments are those of attn_fwd with Sq = 1 and no causal flag (a single new query sees every
 * cached key): q [B, Hq, 1, D], k and v [B, Hkv, Skv, D], o [B, Hq, 1, D] bf16; lse [B, Hq, 1] fp32;
 * all device pointers owned by the caller, 16-byte aligned. Results agree with attn_fwd within
 * rounding (when the partials of the usual work split would not fit, each CTA takes whole
 * (batch, kv head) key ranges instead, which needs none).
 *
 * The first call on a device looks up that device's address of the array (cudaGetSymbolAddress,
 * with the device current); make that first call before any stream capture. With CUDA's lazy
 * module loading (the default since CUDA 12.2) that first call is also when the runtime loads the
 * array onto the device, so the array's memory is taken then: a caller that budgets device memory
 * makes the first call at start-up. Every later call leaves the device's free memory unchanged.
 * Every call on a device shares the array and it keeps the last call's contents; the counters that
 * must start at zero are cleared on `stream` before each launch. Calls that overlap on the GPU
 * (different streams with no ordering between them) race on the array: serialise them. A kernel-side
 * wait that runs out is recorded in the array's status word, which attn_device_status reports.
 *
 * Returns ATTN_OK, an argument error as attn_fwd does, or ATTN_ERR_SCRATCH_LIMIT when the
 * arrival counters alone (one int per (batch, kv head, group of up to 8 query heads)) do not fit in
 * the array, i.e. beyond about two million such triples; nothing is launched then.
 */
#define ATTN_DECODE_NOALLOC_SCRATCH_BYTES (8u << 20) /* 8 MiB */
int attn_decode_noalloc(const void *q, const void *k, const void *v, void *o, float *lse,
                        int B, int Hq, int Hkv, int Skv, int D, float scale, void *stream);

/*
 * attn_decode_paged — single-token decode (Sq == 1) over a paged KV cache whose sequences have
 * different lengths: each sequence attends only to the keys it has filled.
 *
 * Source (page title, section): a KV cache allocated for more tokens than it holds, of which only
 * the filled part is attended to — "第11节：Attention 实现（Flash vs Fallback）", §3 and "Bộ 06 · Bên
 * trong model", Q2 (the cache grows by one token per decode step); decode needs no mask — "AI Infra
 * 入门…", §3. The page layout itself is this library's choice: the pages describe none.
 *
 * Layout (device pointers owned by the caller; bf16 unless noted):
 *   q            [B, Hq, 1, 128]; o [B, Hq, 1, 128]; lse fp32 [B, Hq, 1].
 *   k_pages      [num_pages, Hkv, page_size, 128]: page p of kv head h holds page_size consecutive
 *   v_pages      keys' rows. 16-byte aligned.
 *   block_table  int32 [B, pages_per_seq]: the n-th page_size keys of sequence b live in page
 *                block_table[b * pages_per_seq + n].
 *   seq_lens     int32 [B]: keys filled in sequence b. Each length is clamped to
 *                [0, min(max_seq_len, pages_per_seq * page_size)]; a page index outside
 *                [0, num_pages) reads as zeros. Sequence b attends to keys 0 .. len_b - 1; a
 *                sequence with no keys gets o = 0 and lse = -inf.
 *   max_seq_len  host-side upper bound of the lengths (sizes nothing larger than it needs).
 *   page_size    16, 32, 64 or a multiple of 128.
 *   decode_ctas  CTAs to launch (0: one per resident slot). A performance parameter only.
 * Head dim 128 only; 1 <= B <= 1024; Hq % Hkv == 0. Lengths are read on the device and never on
 * the host, so block_table and seq_lens may be written by earlier work on `stream`.
 * Returns ATTN_OK or a negative attn_status (argument errors before any launch).
 */
int attn_decode_paged(const void *q, const void *k_pages, const void *v_pages, const int *block_table,
                      const int *seq_lens, void *o, float *lse, int B, int Hq, int Hkv, int num_pages,
                      int page_size, int pages_per_seq, int max_seq_len, float scale, int decode_ctas,
                      void *stream);

/*
 * attn_prefill_paged — chunked prefill over a paged, variable-length KV cache: for each sequence b,
 * its Sq new query rows attend to the first len_b keys of its cache, the causal mask aligned to the
 * cache's last Sq keys (query i sees key j iff j <= i + len_b - Sq).
 *
 * Source (page title, section): K = [past K, current K] with the -inf upper triangle on the last
 * seq_len key columns — "第11节：Attention 实现（Flash vs Fallback）", §3; attending only to the filled
 * part of a cache allocated for more tokens — same page, §3, and "Bộ 06 · Bên trong model", Q2–Q3.
 * The cache layout is attn_decode_paged's (this library's choice; the pages describe none).
 *
 *   q            bf16 [B, Hq, Sq, 128] (the new tokens' queries; every sequence has Sq of them).
 *   o, lse       bf16 [B, Hq, Sq, 128] and fp32 [B, Hq, Sq], written entirely.
 *   k_pages, v_pages, block_table, seq_lens, max_seq_len, page_size   as attn_decode_paged: the
 *                new tokens' keys and values must already be in the cache (len_b counts them).
 *   causal       0 or 1. A row that sees no key (len_b < Sq under the mask, or len_b = 0) gets
 *                o = 0 and lse = -inf.
 * Head dim 128 only; Hq % Hkv == 0. Lengths are read on the device, never on the host. Returns
 * ATTN_OK or a negative attn_status (argument errors before any launch).
 */
int attn_prefill_paged(const void *q, const void *k_pages, const void *v_pages, const int *block_table,
                       const int *seq_lens, void *o, float *lse, int B, int Hq, int Hkv, int Sq, int num_pages,
                       int page_size, int pages_per_seq, int max_seq_len, float scale, int causal, void *stream);

/*
 * attn_bwd — backward pass of attn_fwd: given dout = dL/do for a loss L, the gradients
 *   dq = dL/dq [B, Hq, Sq, D], dk = dL/dk and dv = dL/dv [B, Hkv, Skv, D] (bf16, written entirely;
 *   for grouped heads dk and dv sum over the query heads that share a kv head).
 * Inputs are those of the forward call plus its outputs o (bf16 [B, Hq, Sq, D]) and lse (fp32
 * [B, Hq, Sq], natural log), and dout (bf16, layout of o). The softmax weights are recomputed from
 * lse rather than stored — "AI Infra 入门…", §3 (LSE paragraph); the gradients are the derivative of
 * the operation defined at the top of this file. Head dim 128 only; the other sizes, the causal flag
 * and the scale as attn_fwd. The library keeps an fp32 accumulator for dq and two per-row vectors in
 * its workspace (grown stream-ordered like attn_fwd's). Every pointer is a caller-owned device
 * pointer, 16-byte aligned. Returns ATTN_OK or a negative attn_status; never synchronises.
 */
int attn_bwd(const void *q, const void *k, const void *v, const void *o, const void *dout, const float *lse,
             void *dq, void *dk, void *dv, int B, int Hq, int Hkv, int Sq, int Skv, int D,
             float scale, int causal, void *stream);

/*
 * attn_decode_fp8 — single-token decode (Sq == 1) over a K/V cache stored as FP8 (e4m3) codes with
 * one fp32 coefficient per (kv head, channel): the cached key is k~[b,g,j,d] = e4m3(k8[b,g,j,d]) *
 * k_scale[g,d], likewise v~ with v_scale, and the result is attn_fwd's decode over k~, v~.
 *
 * Source (page title, section): "MLA 矩阵乘法吸收的数值稳定性治理", §五 — the KV cache may be kept in
 * FP8 to save bandwidth provided the products accumulate in higher precision (fp32 here, in tensor
 * memory); §二.1 — a coefficient per feature channel. The coefficient's granularity (per kv head and
 * channel, shared by all batch entries) is this library's reading.
 *
 * Layout (device pointers owned by the caller, 16-byte aligned):
 *   q            bf16 [B, Hq, 1, 128]; o bf16 [B, Hq, 1, 128]; lse fp32 [B, Hq, 1] (natural log).
 *   k8, v8       e4m3 codes (1 byte each; the OCP format with bias 7, NaN = S.1111.111)
 *                [B, Hkv, Skv, 128].
 *   k_scale,     fp32 [Hkv, 128].
 *   v_scale
 * The tensor core reads the codes as they are. q * k_scale and the softmax weights enter the
 * products as sums of three e4m3 parts (about 12 significant bits; q is first scaled per head by a
 * power of two into the top of the e4m3 range, which the softmax undoes), so the result matches
 * the dequantised cache to about the accuracy of the bf16 path. Non-finite codes, coefficients or
 * q values give undefined results. Head dim 128 only; Hq % Hkv == 0; decode_ctas as attn_decode_paged.
 * Returns ATTN_OK or a negative attn_status (argument errors before any launch).
 */
int attn_decode_fp8(const void *q, const void *k8, const void *v8, const float *k_scale, const float *v_scale,
                    void *o, float *lse, int B, int Hq, int Hkv, int Skv, int D, float scale, int decode_ctas,
                    void *stream);

/*
 * attn_prefill_fp8 — attn_fwd for any Sq (a prefill of Sq new tokens over a cached prefix, the
 * causal mask aligned to the last Sq keys) over the e4m3 K/V cache of attn_decode_fp8: the result
 * is attn_fwd over k~, v~ (the dequantised cache).
 *
 * Source (page title, section): "MLA 矩阵乘法吸收的数值稳定性治理", §五 (FP8 cache, higher-precision
 * accumulation) and §二.1 (a coefficient per channel); "第11节：Attention 实现（Flash vs Fallback）",
 * §3 (the mask aligned to the last Sq keys).
 *
 * Layout (device pointers owned by the caller, 16-byte aligned): q, o bf16 [B, Hq, Sq, 128];
 * lse fp32 [B, Hq, Sq]; k8, v8 e4m3 codes [B, Hkv, Skv, 128]; k_scale, v_scale fp32 [Hkv, 128].
 * The tensor core reads the codes as they are; q * k_scale (scaled per query row by a power of two
 * into the top of the e4m3 range) enters the score product as a sum of three e4m3 parts (about 12
 * significant bits) and the softmax weights the PV product as a sum of two (about 8, as the bf16
 * path rounds them), with fp32 accumulation in tensor memory, so the result matches the
 * dequantised cache to about the accuracy of the bf16 path. causal 0 or 1; with causal,
 * Sq <= Skv. Head dim 128 only; Hq % Hkv == 0. Non-finite codes, coefficients or q values give
 * undefined results. Returns ATTN_OK or a negative attn_status (argument errors before any launch).
 */
int attn_prefill_fp8(const void *q, const void *k8, const void *v8, const float *k_scale, const float *v_scale,
                     void *o, float *lse, int B, int Hq, int Hkv, int Sq, int Skv, int D, float scale, int causal,
                     void *stream);

/*
 * attn_decode_paged_fp8 — attn_decode_paged over an e4m3 cache: k_pages, v_pages hold e4m3 codes
 * [num_pages, Hkv, page_size, 128] and k_scale, v_scale are as for attn_decode_fp8. Every other
 * argument, rule and return value is attn_decode_paged's.
 */
int attn_decode_paged_fp8(const void *q, const void *k_pages, const void *v_pages, const float *k_scale,
                          const float *v_scale, const int *block_table, const int *seq_lens, void *o, float *lse,
                          int B, int Hq, int Hkv, int num_pages, int page_size, int pages_per_seq, int max_seq_len,
                          float scale, int decode_ctas, void *stream);

/*
 * attn_lse_merge — merges attention over one block of keys into a running result over other keys
 * (the LSE merge of split keys; ring attention calls it once per key block it receives).
 *
 * Source (page title, section): "AI Infra 入门…", §3 (LSE paragraph). Per row, natural logs:
 *   M = max(lse_acc, lse_part), w_a = e^(lse_acc - M), w_p = e^(lse_part - M),
 *   o_acc <- (w_a o_acc + w_p o_part) / (w_a + w_p), lse_acc <- M + ln(w_a + w_p).
 * A side with lse = -inf (no key) has weight 0; a row empty on both sides stays as it is. Start an
 * accumulator at o_acc = 0, lse_acc = -inf.
 *
 * Layout (device pointers owned by the caller, 16-byte aligned): o_acc fp32 [rows, D] and lse_acc
 * fp32 [rows], updated in place; o_part bf16 [rows, D] and lse_part fp32 [rows] (an attn_fwd
 * result); o_out bf16 [rows, D] or NULL: when given, also receives the merged O rounded to bf16.
 * rows = B * Hq * Sq of the attention call; D in {32, 64, 128}. rows = 0 launches nothing.
 * Returns ATTN_OK or a negative attn_status (argument errors before any launch); never allocates.
 */
int attn_lse_merge(float *o_acc, float *lse_acc, const void *o_part, const float *lse_part, void *o_out,
                   long long rows, int D, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_ATTN_H */
