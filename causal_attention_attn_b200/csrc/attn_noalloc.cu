/*
 * attn_noalloc.cu — single-token decode that allocates nothing.
 *
 * attn_fwd keeps the decode kernel's split partials and arrival counters in a workspace that the
 * library grows with cudaMalloc on first use. Some callers cannot allow that: cudaMalloc can
 * synchronise the whole device and take milliseconds, which a latency-bound serving loop cannot
 * absorb mid-request, and some processes hand all device memory to one allocator at start-up (a
 * framework's caching allocator or a fixed memory budget), so an allocation made behind that
 * allocator's back either fails or breaks its accounting. attn_decode_noalloc serves those callers:
 * the scratch lives in a fixed-size array in the library's own device memory, and the call makes no
 * allocation and frees nothing. The runtime places the array on a device when it loads this file's
 * module there; with lazy module loading (the CUDA 12.2+ default) that happens at the first
 * cudaGetSymbolAddress below, i.e. in the first call on each device, so a caller that budgets
 * device memory makes that first call at start-up. A kernel-side wait that runs out is recorded in
 * the array's status word, which attn_device_status reads and clears.
 *
 * The array is shared by every call on a device and keeps the last call's contents. The arrival
 * counters, which must start at zero, are cleared on the stream before each launch; calls that
 * overlap on the GPU (different streams, no ordering between them) race on the array and must be
 * serialised by the caller.
 */
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "attn.h"
#include "kernels.h"

namespace attn_b200 {
namespace {

constexpr size_t kScratchBytes = ATTN_DECODE_NOALLOC_SCRATCH_BYTES;
constexpr size_t kStatusBytes = 256;  // status word, padded to keep what follows 256-byte aligned

// Decode scratch: [status word | arrival counters | split partials]. Every GPU that loads the
// library holds these bytes until the process exits. Host code must not use this symbol as an
// address: it is a host-side stand-in; the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

std::mutex g_setup_mutex;
unsigned char *g_scratch_addr[kMaxDevices];  // device address of g_decode_scratch, per device

// Once per device, with that device current: look up this device's address of the array.
int scratch_for_current_device(unsigned char **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_scratch_addr[dev] == nullptr) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess || ptr == nullptr) {
            cudaGetLastError();
            return ATTN_ERR_CUDA;
        }
        g_scratch_addr[dev] = static_cast<unsigned char *>(ptr);
    }
    *out = g_scratch_addr[dev];
    return ATTN_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

int *noalloc_status_word()
{
    const int dev = current_device_index();
    if (dev < 0)
        return nullptr;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    return reinterpret_cast<int *>(g_scratch_addr[dev]);
}

}  // namespace attn_b200

using namespace attn_b200;

extern "C" int attn_decode_noalloc(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq,
                                   int Hkv, int Skv, int D, float scale, void *stream_ptr)
{
    if (!q || !k || !v || !o || !lse)
        return ATTN_ERR_NULL;
    if (B < 1 || Hq < 1 || Hkv < 1 || Skv < 1)
        return ATTN_ERR_SHAPE;
    if (Hq % Hkv != 0)
        return ATTN_ERR_GQA;
    if (D != 32 && D != 64 && D != 128)
        return ATTN_ERR_HEADDIM;
    if (static_cast<long long>(B) * Hq > INT_MAX || static_cast<long long>(B) * Hkv * Skv > INT_MAX)
        return ATTN_ERR_SHAPE;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return ATTN_ERR_ALIGN;
    if (!(scale > 0.f) || !std::isfinite(scale))
        return ATTN_ERR_SCALE;

    // Same work split as attn_fwd (this also checks that the device is an sm_100 part); if the
    // shared-pair partials do not fit, one CTA per pair needs none.
    const int ctas = attn_decode_ctas(B, Hq, Hkv, Skv, D);
    if (ctas < 0)
        return ctas;
    int sm_count = 0, dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
    }
    DecodePlan plan;
    if (decode_plan(B, Hq, Hkv, Skv, D, ctas, sm_count, &plan) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_SHAPE;
    }
    const size_t counter_bytes = ((static_cast<size_t>(plan.pairs) * sizeof(int) + 255) / 256) * 256;
    if (kStatusBytes + counter_bytes > kScratchBytes)
        return ATTN_ERR_SCRATCH_LIMIT;
    const size_t partial_room = (kScratchBytes - kStatusBytes - counter_bytes) / sizeof(float);
    if (plan.partial_floats > partial_room) {
        if (decode_plan(B, Hq, Hkv, Skv, D, static_cast<int>(plan.pairs), sm_count, &plan) != cudaSuccess ||
            plan.partial_floats > partial_room) {
            cudaGetLastError();
            return ATTN_ERR_SCRATCH_LIMIT;
        }
    }

    unsigned char *scratch = nullptr;
    const int rc = scratch_for_current_device(&scratch);
    if (rc != ATTN_OK)
        return rc;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
    int *counters = reinterpret_cast<int *>(scratch + kStatusBytes);
    float *partials = reinterpret_cast<float *>(scratch + kStatusBytes + counter_bytes);
    if (cudaMemsetAsync(counters, 0, static_cast<size_t>(plan.pairs) * sizeof(int), stream) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
    }

    DecodeArgs a;
    a.q = q;
    a.k = k;
    a.v = v;
    a.o = o;
    a.lse = lse;
    a.B = B;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.Skv = Skv;
    a.D = D;
    a.scale = scale;
    a.plan = plan;
    a.ws = partials;
    a.counters = counters;
    a.status = reinterpret_cast<int *>(scratch);
    if (launch_decode(a, stream) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_LAUNCH;
    }
    return ATTN_OK;
}
