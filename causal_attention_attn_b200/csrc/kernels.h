/*
 * kernels.h — internal launch interface between the C-ABI layer (attn_api.cu) and the two kernels.
 * Not part of the public ABI.
 */
#pragma once

#include <cuda_runtime.h>

namespace attn_b200 {

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
};

struct PrefillArgs {
    const void *q, *k, *v;
    void *o;
    float *lse;
    int B, Hq, Hkv, Sq, Skv, D;
    float scale;
    int causal;
    int *status;  // device status word
};

struct DecodeArgs {
    const void *q, *k, *v;
    void *o;
    float *lse;
    int B, Hq, Hkv, Skv, D;
    float scale;
    int splits;         // >= 1, already clamped so that every split is non-empty
    float *ws_o;        // [B*Hq*splits*D] partial outputs (only when splits > 1)
    float *ws_lse;      // [B*Hq*splits] partial log2-sum-exp (only when splits > 1)
    int *counters;      // [B*Hkv*head_groups] arrival counters, zero between calls
    int *status;        // device status word
};

// Returns a cudaError_t value (cudaSuccess on success); never synchronises.
cudaError_t launch_prefill(const PrefillArgs &a, cudaStream_t stream, int *encode_error);

// Decode geometry shared by the host planner and the launcher.
int decode_heads_per_cta(int group);           // G: 1, 2, 4 or 8
int decode_keys_per_chunk(int group);          // keys per pipeline stage
int decode_effective_splits(int Skv, int group, int requested);  // clamp so that no split is empty
cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream);
int decode_ctas_per_sm(int D, int group);      // occupancy of the decode kernel (>= 1)

}  // namespace attn_b200
