/*
 * kernels.h — internal launch interface between the C-ABI layer (attn_api.cu) and the two kernels.
 * Not part of the public ABI.
 */
#pragma once

#include <cuda_runtime.h>

namespace attn_b200 {

// Devices the library keeps state for (function attributes, occupancy, workspaces), by index.
constexpr int kMaxDevices = 64;

// Index of the current device, or -1 if it cannot be read or is kMaxDevices or beyond. Function
// attributes such as the dynamic shared-memory limit take effect on the device that is current
// when they are set, so the launchers keep them per device.
inline int current_device_index()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return -1;
    }
    return (dev >= 0 && dev < kMaxDevices) ? dev : -1;
}

// Device status word values: 0 = fine, otherwise the site of the first wait that ran out.
enum WaitSite : int {
    kSiteNone = 0,
    kSitePrefillTmaEmpty = 1,
    kSitePrefillMmaQ = 2,
    kSitePrefillMmaFull = 3,
    kSitePrefillMmaSFree = 4,
    kSitePrefillMmaPFull = 5,
    kSitePrefillSoftmaxSFull = 6,
    kSitePrefillSoftmaxODone = 7,
    kSitePrefillEpilogue = 8,
    kSitePrefillDrain = 9,
    kSiteDecodeProducer = 16,
    kSiteDecodeConsumer = 17,
    kSiteBwd = 24,
    kSiteFp8Prefill = 32,
};

// Element strides of a [batch][head][row][dim] tensor with a contiguous dim (see tma_host.h).
struct TensorStrides {
    long long b, h, s;
};

struct PrefillArgs {
    const void *q, *k, *v;
    void *o;
    float *lse;  // [B][Hq][Sq], contiguous
    int B, Hq, Hkv, Sq, Skv, D;
    float scale;
    int causal;
    int *status;       // device status word
    int sm_count = 0;  // SMs of the device: the persistent grid's size
    TensorStrides qs, ks, vs, os;  // element strides of q, k, v, o
    // Paged, variable-length cache (seq_lens != nullptr; head dim 128): k, v are
    // [num_pages][Hkv][page_size][D]; sequence b holds min(max(seq_lens[b], 0), cap) keys, cap =
    // min(max_seq_len, pages_per_seq * page_size), in pages block_table[b][...]; Skv is unused.
    const int *seq_lens = nullptr;
    const int *block_table = nullptr;
    int num_pages = 0, page_size = 0, pages_per_seq = 0, max_seq_len = 0;
};

// How a decode (Sq == 1) is spread over persistent CTAs. A "pair" is one (batch, kv head, group of
// G query heads); its keys are cut into `cpp` chunks of `ck` keys; CTA c of `ctas` takes units
// [c*total/ctas, (c+1)*total/ctas) of the pairs' chunks laid end to end.
struct DecodePlan {
    int G;                  // query heads per pair
    int head_groups;        // (Hq / Hkv) / G
    long long pairs;        // B * Hkv * head_groups
    int ck;                 // keys per chunk
    int cpp;                // chunks per pair
    long long total;        // pairs * cpp
    int ctas;               // CTAs launched
    int max_contrib;        // most CTAs that can share one pair
    size_t partial_floats;  // workspace floats for shared pairs' partials (0 if no pair is shared)
};

struct DecodeArgs {
    const void *q, *k, *v;
    void *o;
    float *lse;
    // Element strides of q, k, v and o (dense cache, tensor-core kernel); `strided` false: the
    // contiguous [B][H][S][D] layouts, which the CUDA-core kernel requires.
    bool strided = false;
    TensorStrides qs{}, ks{}, vs{}, os{};
    int B, Hq, Hkv, Skv, D;
    float scale;
    DecodePlan plan;
    float *ws;          // plan.partial_floats floats (may be null when that is 0)
    int *counters;      // plan.pairs arrival counters, zero between calls
    int *status;        // device status word
    // Paged, variable-length cache (tensor-core decode only; seq_lens == nullptr: the dense cache
    // above). k, v are then [num_pages][Hkv][page_size][D]; block_table [B][pages_per_seq] and
    // seq_lens [B] are device int32 arrays; lengths are clamped to [0, min(max_seq_len, capacity)].
    const int *seq_lens = nullptr;
    const int *block_table = nullptr;
    int num_pages = 0, page_size = 0, pages_per_seq = 0, max_seq_len = 0;
    // e4m3 cache (tensor-core decode only): k, v hold e4m3 codes; k_scale, v_scale are device fp32
    // [Hkv][D] coefficients (value = code * coefficient of its kv head and channel).
    bool fp8 = false;
    const float *k_scale = nullptr, *v_scale = nullptr;
};

// Returns a cudaError_t value (cudaSuccess on success); never synchronises.
cudaError_t launch_prefill(const PrefillArgs &a, cudaStream_t stream, int *encode_error);

// Prefill over an e4m3 K/V cache (head dim 128): k8, v8 [B][Hkv][Skv][D] codes, k_scale, v_scale
// [Hkv][D] fp32 coefficients; q, o [B][Hq][Sq][D] bf16, lse [B][Hq][Sq]; contiguous.
struct PrefillFp8Args {
    const void *q, *k8, *v8;
    const float *k_scale, *v_scale;
    void *o;
    float *lse;
    int B, Hq, Hkv, Sq, Skv, D;
    float scale;
    int causal;
    int *status;  // device status word
};
cudaError_t launch_prefill_fp8(const PrefillFp8Args &a, cudaStream_t stream, int *encode_error);

// Backward pass (head dim 128): dq, dk, dv from q, k, v, o, dout and the forward's lse.
struct BwdArgs {
    const void *q, *k, *v, *o, *dout;
    const float *lse;
    void *dq, *dk, *dv;
    int B, Hq, Hkv, Sq, Skv, D;
    float scale;
    int causal;
    void *ws;      // bwd_workspace_bytes(B, Hq, Sq, D) bytes, 256-byte aligned
    int *status;   // device status word
    int sm_count;  // SMs of the device (chooses the head split)
};
size_t bwd_workspace_bytes(int B, int Hq, int Sq, int D);
cudaError_t launch_bwd(const BwdArgs &a, cudaStream_t stream, int *encode_error);

// LSE merge of a partial result (bf16 o_part, fp32 lse_part) into an fp32 accumulator, rows x D
// (D in {32, 64, 128}); o_out (bf16, may be null) receives the merged O.
cudaError_t launch_lse_merge(float *o_acc, float *lse_acc, const void *o_part, const float *lse_part, void *o_out,
                             long long rows, int D, int sm_count, cudaStream_t stream);

// Decode planning and launch. requested_ctas <= 0 means one CTA per resident slot on the device.
int decode_heads_per_cta(int group, int D);  // G: 1, 2, 4 or 8 (up to 16 for D = 128)
// fp8: plan for the e4m3-cache variant of the tensor-core kernel (its own occupancy).
cudaError_t decode_plan(int B, int Hq, int Hkv, int Skv, int D, int requested_ctas, int sm_count, DecodePlan *plan,
                        bool fp8 = false);
cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream);

// Head dim 128 decodes on the tensor core (decode_tc_sm100.cu); launch_decode routes there.
int decode_tc_heads_per_pair(int group);  // G: largest power of two dividing the group, at most 16
int decode_tc_chunk_keys();               // keys per chunk (128)
cudaError_t decode_tc_ctas_per_sm(int G, bool fp8, int *ctas_per_sm);
size_t decode_tc_partial_floats(int G, int ctas);  // workspace floats for shared pairs' partials
constexpr int kPagedMaxBatch = 1024;  // batch entries a paged decode may have (per-CTA scan in shared memory)
// Plan of a paged, variable-length decode: lengths are only known on the device, so the plan holds
// upper bounds (cpp from max_seq_len; total is computed by each CTA); every pair may be shared.
cudaError_t decode_plan_paged(int B, int Hq, int Hkv, int max_seq_len, int requested_ctas, int sm_count,
                              DecodePlan *plan, bool fp8 = false);
cudaError_t launch_decode_tc(const DecodeArgs &a, cudaStream_t stream);

// The status word of attn_decode_noalloc's fixed scratch array on the current device, or nullptr
// if that entry point has not run on it (its address is only looked up by its first call there).
int *noalloc_status_word();

}  // namespace attn_b200
