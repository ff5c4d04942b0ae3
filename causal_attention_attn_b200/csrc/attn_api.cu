/*
 * attn_api.cu — the C ABI declared in include/attn.h: argument validation, dispatch between the
 * prefill and decode kernels, the per-device workspace, and status reporting. No arithmetic of the
 * method happens here; every step runs in the two kernels.
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

constexpr int kVersion = 700;  // 0.7.0: attn_prefill_fp8 (prefill over an e4m3 K/V cache); 0.6.0: attn_fwd_host

struct DeviceState {
    bool probed = false;
    bool supported = false;
    int sm_count = 0;
    void *block = nullptr;  // status word + counters + partials, one allocation
    size_t bytes = 0;
    int *status = nullptr;
    int *counters = nullptr;
    size_t counter_count = 0;
    float *partials = nullptr;
    size_t partial_floats = 0;
    void *bwd_block = nullptr;  // backward pass: dq accumulator and per-row vectors
    size_t bwd_bytes = 0;
    // attn_fwd_host: a stream for the copies in, one for the copies out, and the events that order
    // them against the caller's stream (created on first use, kept for the process).
    cudaStream_t copy_in = nullptr, copy_out = nullptr;
    cudaEvent_t ev_start = nullptr, ev_in = nullptr, ev_done = nullptr, ev_out = nullptr;
};

std::mutex g_mutex;
DeviceState g_dev[kMaxDevices];
// attn_fwd_host: the copy streams and the events are shared by all calls on a device, so one call
// queues its whole pipeline before the next starts (the events are re-recorded per slice).
std::mutex g_host_mutex;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int validate(const void *q, const void *k, const void *v, const void *o, const float *lse, int B, int Hq, int Hkv,
             int Sq, int Skv, int D, float scale, int causal)
{
    if (!q || !k || !v || !o || !lse)
        return ATTN_ERR_NULL;
    if (B < 1 || Hq < 1 || Hkv < 1 || Sq < 1 || Skv < 1 || D < 1)
        return ATTN_ERR_SHAPE;
    if (Hq % Hkv != 0)
        return ATTN_ERR_GQA;
    if (D != 32 && D != 64 && D != 128)
        return ATTN_ERR_HEADDIM;
    // Flat row indices (b*H + h)*S + i must fit in a 32-bit int.
    if (static_cast<long long>(B) * Hq * Sq > INT_MAX || static_cast<long long>(B) * Hkv * Skv > INT_MAX)
        return ATTN_ERR_SHAPE;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return ATTN_ERR_ALIGN;
    if (causal != 0 && causal != 1)
        return ATTN_ERR_SHAPE;
    if (causal && Sq > Skv)
        return ATTN_ERR_CAUSAL_SQ_GT_SKV;
    if (!(scale > 0.f) || !std::isfinite(scale))
        return ATTN_ERR_SCALE;
    return ATTN_OK;
}

// Probe the current device once; returns the state or nullptr with *err set.
DeviceState *device_state(int *err)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        *err = ATTN_ERR_CUDA;
        return nullptr;
    }
    DeviceState &s = g_dev[dev];
    if (!s.probed) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            *err = ATTN_ERR_CUDA;
            return nullptr;
        }
        s.supported = (major == 10 && minor == 0);
        s.sm_count = sms;
        s.probed = true;
    }
    if (!s.supported) {
        *err = ATTN_ERR_ARCH;
        return nullptr;
    }
    return &s;
}

// Make sure the workspace holds `counters` ints and `partials` floats (plus the status word).
// Growth is stream-ordered: the new block comes from the device's stream-ordered pool on `stream`
// (cudaMallocAsync), is cleared there, and the old block is released on `stream` after the work
// already queued on it (cudaFreeAsync). Nothing waits on the host. A status word that a kernel set in
// the old block (a wait that ran out) is carried into the new one on the stream.
int ensure_workspace(DeviceState &s, size_t counters, size_t partials, cudaStream_t stream)
{
    if (s.block && counters <= s.counter_count && partials <= s.partial_floats)
        return ATTN_OK;
    size_t nc = counters > s.counter_count ? counters : s.counter_count;
    size_t np = partials > s.partial_floats ? partials : s.partial_floats;
    if (nc < 1024)
        nc = 1024;
    const size_t head = 256;  // status word, padded
    const size_t cbytes = ((nc * sizeof(int) + 255) / 256) * 256;
    const size_t bytes = head + cbytes + np * sizeof(float);
    void *block = nullptr;
    if (cudaMallocAsync(&block, bytes, stream) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_WORKSPACE;
    }
    if (cudaMemsetAsync(block, 0, head + cbytes, stream) != cudaSuccess ||
        (s.block && cudaMemcpyAsync(block, s.block, sizeof(int), cudaMemcpyDeviceToDevice, stream) != cudaSuccess)) {
        cudaGetLastError();
        cudaFreeAsync(block, stream);
        cudaGetLastError();
        return ATTN_ERR_WORKSPACE;
    }
    if (s.block && cudaFreeAsync(s.block, stream) != cudaSuccess)
        cudaGetLastError();  // the old block stays allocated; nothing reads it any more
    s.block = block;
    s.bytes = bytes;
    s.status = static_cast<int *>(block);
    s.counters = reinterpret_cast<int *>(static_cast<char *>(block) + head);
    s.counter_count = nc;
    s.partials = reinterpret_cast<float *>(static_cast<char *>(block) + head + cbytes);
    s.partial_floats = np;
    return ATTN_OK;
}

// The copy streams and events of attn_fwd_host, created once per device (under g_mutex).
int ensure_host_pipeline(DeviceState &s)
{
    if (s.ev_out)
        return ATTN_OK;
    if (!s.copy_in && cudaStreamCreateWithFlags(&s.copy_in, cudaStreamNonBlocking) != cudaSuccess)
        s.copy_in = nullptr;
    if (s.copy_in && !s.copy_out && cudaStreamCreateWithFlags(&s.copy_out, cudaStreamNonBlocking) != cudaSuccess)
        s.copy_out = nullptr;
    cudaEvent_t *evs[4] = {&s.ev_start, &s.ev_in, &s.ev_done, &s.ev_out};
    bool ok = s.copy_in && s.copy_out;
    for (cudaEvent_t *e : evs)
        if (ok && !*e && cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess) {
            *e = nullptr;
            ok = false;
        }
    if (!ok) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
    }
    return ATTN_OK;
}

// Element strides (batch, head, row) of q, k, v and o; `strided` false: the contiguous layouts.
struct Layouts {
    TensorStrides q, k, v, o;
    bool strided;
};

Layouts contiguous_layouts(int Hq, int Hkv, int Sq, int Skv, int D)
{
    Layouts L;
    L.q = L.o = TensorStrides{static_cast<long long>(Hq) * Sq * D, static_cast<long long>(Sq) * D, D};
    L.k = L.v = TensorStrides{static_cast<long long>(Hkv) * Skv * D, static_cast<long long>(Skv) * D, D};
    L.strided = false;
    return L;
}

int run(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq, int Hkv, int Sq, int Skv,
        int D, float scale, int causal, int decode_ctas, const Layouts &st, void *stream_ptr)
{
    int rc = validate(q, k, v, o, lse, B, Hq, Hkv, Sq, Skv, D, scale, causal);
    if (rc != ATTN_OK)
        return rc;
    if (decode_ctas < 0)
        return ATTN_ERR_SHAPE;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
    std::lock_guard<std::mutex> lock(g_mutex);
    int err = ATTN_OK;
    DeviceState *s = device_state(&err);
    if (!s)
        return err;

    // Sq == 1 runs a decode kernel: the tensor-core one (D = 128) takes any layout, the CUDA-core one
    // (D = 32, 64) only the contiguous one; a strided decode with D < 128 runs the prefill kernel.
    if (Sq == 1 && (D == 128 || !st.strided)) {
        DecodePlan plan;
        if (decode_plan(B, Hq, Hkv, Skv, D, decode_ctas, s->sm_count, &plan) != cudaSuccess) {
            cudaGetLastError();
            return ATTN_ERR_SHAPE;
        }
        rc = ensure_workspace(*s, static_cast<size_t>(plan.pairs), plan.partial_floats, stream);
        if (rc != ATTN_OK)
            return rc;
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
        a.ws = s->partials;
        a.counters = s->counters;
        a.status = s->status;
        a.strided = st.strided;
        a.qs = st.q;
        a.ks = st.k;
        a.vs = st.v;
        a.os = st.o;
        if (launch_decode(a, stream) != cudaSuccess) {
            cudaGetLastError();
            return ATTN_ERR_LAUNCH;
        }
        return ATTN_OK;
    }

    rc = ensure_workspace(*s, 0, 0, stream);
    if (rc != ATTN_OK)
        return rc;
    PrefillArgs a;
    a.q = q;
    a.k = k;
    a.v = v;
    a.o = o;
    a.lse = lse;
    a.B = B;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.Sq = Sq;
    a.Skv = Skv;
    a.D = D;
    a.scale = scale;
    a.causal = causal;
    a.status = s->status;
    a.sm_count = s->sm_count;
    a.qs = st.q;
    a.ks = st.k;
    a.vs = st.v;
    a.os = st.o;
    int encode_error = 0;
    const cudaError_t e = launch_prefill(a, stream, &encode_error);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return encode_error != 0 ? ATTN_ERR_CUDA : ATTN_ERR_LAUNCH;
    }
    return ATTN_OK;
}

}  // namespace
}  // namespace attn_b200

using namespace attn_b200;

extern "C" int attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq, int Hkv,
                        int Sq, int Skv, int D, float scale, int causal, void *stream)
{
    return run(q, k, v, o, lse, B, Hq, Hkv, Sq, Skv, D, scale, causal, 0, contiguous_layouts(Hq, Hkv, Sq, Skv, D),
               stream);
}

extern "C" int attn_fwd_ex(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq,
                           int Hkv, int Sq, int Skv, int D, float scale, int causal, int decode_ctas, void *stream)
{
    return run(q, k, v, o, lse, B, Hq, Hkv, Sq, Skv, D, scale, causal, decode_ctas,
               contiguous_layouts(Hq, Hkv, Sq, Skv, D), stream);
}

extern "C" int attn_fwd_host(const void *q_host, const void *k_host, const void *v_host, void *o_host,
                             float *lse_host, void *q_dev, void *k_dev, void *v_dev, void *o_dev, float *lse_dev,
                             int B, int Hq, int Hkv, int Sq, int Skv, int D, float scale, int causal, void *stream_ptr)
{
    if (!q_host || !k_host || !v_host || !o_host || !lse_host)
        return ATTN_ERR_NULL;
    int rc = validate(q_dev, k_dev, v_dev, o_dev, lse_dev, B, Hq, Hkv, Sq, Skv, D, scale, causal);
    if (rc != ATTN_OK)
        return rc;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
    std::lock_guard<std::mutex> host_lock(g_host_mutex);
    cudaStream_t s_in, s_out;
    cudaEvent_t ev_start, ev_in, ev_done, ev_out;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        int err = ATTN_OK;
        DeviceState *s = device_state(&err);
        if (!s)
            return err;
        if ((rc = ensure_host_pipeline(*s)) != ATTN_OK)
            return rc;
        s_in = s->copy_in;
        s_out = s->copy_out;
        ev_start = s->ev_start;
        ev_in = s->ev_in;
        ev_done = s->ev_done;
        ev_out = s->ev_out;
    }
    // A unit is one (batch, kv head) with its group of query heads; its q, k, v, o and lse rows are
    // contiguous, so a run of units is one copy per tensor and one attention call over B' = units,
    // Hq' = group, Hkv' = 1. Slice boundaries fall on whole 16-byte blocks of lse.
    const int group = Hq / Hkv;
    const long long units = static_cast<long long>(B) * Hkv;
    long long align = 1;
    while ((static_cast<long long>(group) * Sq * align) % 4 != 0)
        align *= 2;
    constexpr long long kSlices = 8;
    const size_t q_head = static_cast<size_t>(Sq) * D * 2, kv_unit = static_cast<size_t>(Skv) * D * 2;
    // A slice: the query heads [a, b) of the flat (unit, head) order, which cover the units
    // [a / group, (b - 1) / group]; either whole units or one half of one unit.
    struct Slice {
        long long a, b;
    };
    Slice slices[kSlices + 2];
    int n_slices = 0;
    // The pipeline's fill (the first slice's copy in) and drain (the last slice's attention and copy
    // out) are not overlapped: with few units the first and the last unit go in halves (of its query
    // heads; the first half also brings the unit's K and V), which shortens both.
    // (Half a group of Sq rows is then a whole number of 16-byte blocks of lse, and so is every unit.)
    const bool halves = units >= 2 && group % 2 == 0 && (static_cast<long long>(group / 2) * Sq) % 4 == 0;
    if (halves) {
        const long long g = group, h = group / 2;
        slices[n_slices++] = {0, h};
        slices[n_slices++] = {h, g};
        const long long mid = units - 2;  // whole units 1 .. units - 2, in up to kSlices - 2 slices
        long long m0 = 0;
        for (long long i = 1; i <= kSlices - 2 && m0 < mid; ++i) {
            const long long m1 = mid * i / (kSlices - 2);
            if (m1 <= m0)
                continue;
            slices[n_slices++] = {(1 + m0) * g, (1 + m1) * g};
            m0 = m1;
        }
        slices[n_slices++] = {(units - 1) * g, (units - 1) * g + h};
        slices[n_slices++] = {(units - 1) * g + h, units * g};
    } else {
        long long u0 = 0;
        for (long long i = 1; i <= kSlices && u0 < units; ++i) {
            const long long u1 = (i == kSlices) ? units : (units * i / kSlices) / align * align;
            if (u1 <= u0)
                continue;
            slices[n_slices++] = {u0 * group, u1 * group};
            u0 = u1;
        }
    }
    auto at = [](const void *p, size_t off) { return static_cast<const char *>(p) + off; };
    auto atw = [](void *p, size_t off) { return static_cast<char *>(p) + off; };
    // The copy streams start after the work already queued on `stream` (which may still use the
    // device buffers), and `stream` continues after the last copy out.
    if (cudaEventRecord(ev_start, stream) != cudaSuccess || cudaStreamWaitEvent(s_in, ev_start, 0) != cudaSuccess ||
        cudaStreamWaitEvent(s_out, ev_start, 0) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
    }
    long long kv_done = 0;  // units whose K and V have been queued for copying in
    for (int i = 0; i < n_slices && rc == ATTN_OK; ++i) {
        const long long a = slices[i].a, b = slices[i].b;
        const long long u0 = a / group, u1 = (b - 1) / group + 1;
        const bool whole = a % group == 0 && b % group == 0;
        const size_t qo = static_cast<size_t>(a) * q_head, qn = static_cast<size_t>(b - a) * q_head;
        const size_t lo = static_cast<size_t>(a) * Sq, ln = static_cast<size_t>(b - a) * Sq;
        if (cudaMemcpyAsync(atw(q_dev, qo), at(q_host, qo), qn, cudaMemcpyHostToDevice, s_in) != cudaSuccess) {
            cudaGetLastError();
            rc = ATTN_ERR_CUDA;
            break;
        }
        if (kv_done < u1) {
            const size_t ko = static_cast<size_t>(kv_done) * kv_unit, kn = static_cast<size_t>(u1 - kv_done) * kv_unit;
            if (cudaMemcpyAsync(atw(k_dev, ko), at(k_host, ko), kn, cudaMemcpyHostToDevice, s_in) != cudaSuccess ||
                cudaMemcpyAsync(atw(v_dev, ko), at(v_host, ko), kn, cudaMemcpyHostToDevice, s_in) != cudaSuccess) {
                cudaGetLastError();
                rc = ATTN_ERR_CUDA;
                break;
            }
            kv_done = u1;
        }
        if (cudaEventRecord(ev_in, s_in) != cudaSuccess || cudaStreamWaitEvent(stream, ev_in, 0) != cudaSuccess) {
            cudaGetLastError();
            rc = ATTN_ERR_CUDA;
            break;
        }
        const size_t ku = static_cast<size_t>(u0) * kv_unit;
        const int nb = whole ? static_cast<int>(u1 - u0) : 1, nh = whole ? group : static_cast<int>(b - a);
        rc = run(at(q_dev, qo), at(k_dev, ku), at(v_dev, ku), atw(o_dev, qo), lse_dev + lo, nb, nh, 1, Sq, Skv, D, scale,
                 causal, 0, contiguous_layouts(nh, 1, Sq, Skv, D), stream);
        if (rc != ATTN_OK)
            break;
        if (cudaEventRecord(ev_done, stream) != cudaSuccess || cudaStreamWaitEvent(s_out, ev_done, 0) != cudaSuccess ||
            cudaMemcpyAsync(atw(o_host, qo), at(o_dev, qo), qn, cudaMemcpyDeviceToHost, s_out) != cudaSuccess ||
            cudaMemcpyAsync(lse_host + lo, lse_dev + lo, ln * sizeof(float), cudaMemcpyDeviceToHost, s_out) !=
                cudaSuccess) {
            cudaGetLastError();
            rc = ATTN_ERR_CUDA;
            break;
        }
    }
    // Join the copy streams back into `stream` on every path, so that later work on it (or a
    // synchronisation of it) covers everything this call queued.
    if (cudaEventRecord(ev_in, s_in) != cudaSuccess || cudaStreamWaitEvent(stream, ev_in, 0) != cudaSuccess ||
        cudaEventRecord(ev_out, s_out) != cudaSuccess || cudaStreamWaitEvent(stream, ev_out, 0) != cudaSuccess) {
        cudaGetLastError();
        if (rc == ATTN_OK)
            rc = ATTN_ERR_CUDA;
    }
    return rc;
}

namespace {

// A stride triple the kernels can use: every stride >= 1, a whole number of 16-byte units (8 bf16
// elements: the TMA and the 16-byte output stores need it) and below 2^38 elements.
bool strides_ok(const long long *st)
{
    for (int i = 0; i < 3; ++i)
        if (st[i] < 1 || st[i] % 8 != 0 || st[i] >= (1LL << 38))
            return false;
    return true;
}

}  // namespace

extern "C" int attn_fwd_strided(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq,
                                int Hkv, int Sq, int Skv, int D, const long long *q_strides, const long long *k_strides,
                                const long long *v_strides, const long long *o_strides, float scale, int causal,
                                void *stream)
{
    if (!q_strides || !k_strides || !v_strides || !o_strides)
        return ATTN_ERR_NULL;
    if (!strides_ok(q_strides) || !strides_ok(k_strides) || !strides_ok(v_strides) || !strides_ok(o_strides))
        return ATTN_ERR_ALIGN;
    Layouts L;
    L.q = TensorStrides{q_strides[0], q_strides[1], q_strides[2]};
    L.k = TensorStrides{k_strides[0], k_strides[1], k_strides[2]};
    L.v = TensorStrides{v_strides[0], v_strides[1], v_strides[2]};
    L.o = TensorStrides{o_strides[0], o_strides[1], o_strides[2]};
    L.strided = true;
    return run(q, k, v, o, lse, B, Hq, Hkv, Sq, Skv, D, scale, causal, 0, L, stream);
}

extern "C" int attn_decode_ctas(int B, int Hq, int Hkv, int Skv, int D)
{
    if (B < 1 || Hq < 1 || Hkv < 1 || Skv < 1)
        return ATTN_ERR_SHAPE;
    if (Hq % Hkv != 0)
        return ATTN_ERR_GQA;
    if (D != 32 && D != 64 && D != 128)
        return ATTN_ERR_HEADDIM;
    std::lock_guard<std::mutex> lock(g_mutex);
    int err = ATTN_OK;
    DeviceState *s = device_state(&err);
    if (!s)
        return err;
    DecodePlan plan;
    if (decode_plan(B, Hq, Hkv, Skv, D, 0, s->sm_count, &plan) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_SHAPE;
    }
    return plan.ctas;
}

extern "C" const char *attn_status_string(int status)
{
    switch (status) {
    case ATTN_OK:
        return "ok";
    case ATTN_ERR_NULL:
        return "a required pointer is NULL";
    case ATTN_ERR_SHAPE:
        return "invalid size: every size must be >= 1, causal must be 0 or 1, and flat row indices must fit in int32";
    case ATTN_ERR_GQA:
        return "Hq must be a multiple of Hkv";
    case ATTN_ERR_HEADDIM:
        return "unsupported head dim: D must be 32, 64 or 128";
    case ATTN_ERR_ALIGN:
        return "every pointer must be 16-byte aligned";
    case ATTN_ERR_CAUSAL_SQ_GT_SKV:
        return "causal attention needs Sq <= Skv (the mask covers the last Sq keys)";
    case ATTN_ERR_ARCH:
        return "the current device is not an sm_100 (B200-class) GPU";
    case ATTN_ERR_WORKSPACE:
        return "could not allocate the library workspace";
    case ATTN_ERR_LAUNCH:
        return "kernel launch failed";
    case ATTN_ERR_DEVICE_TIMEOUT:
        return "a kernel-side wait ran out of time; the results of that call are invalid";
    case ATTN_ERR_SCALE:
        return "scale must be finite and > 0";
    case ATTN_ERR_CUDA:
        return "a CUDA runtime call failed";
    case ATTN_ERR_SCRATCH_LIMIT:
        return "the decode needs more scratch than the fixed no-allocation buffer holds "
               "(too many (batch, kv head, head group) work units for attn_decode_noalloc)";
    default:
        return "unknown status";
    }
}

extern "C" int attn_version(void) { return kVersion; }

extern "C" int attn_device_status(void *stream_ptr)
{
    cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
    std::lock_guard<std::mutex> lock(g_mutex);
    int err = ATTN_OK;
    DeviceState *s = device_state(&err);
    if (!s)
        return err;
    // Two status words: the workspace's (every entry point but attn_decode_noalloc) and the one at
    // the start of attn_decode_noalloc's fixed array (once that entry point has run on this device).
    int *words[2] = {s->block ? s->status : nullptr, noalloc_status_word()};
    bool timed_out = false;
    for (int *word : words) {
        if (!word)
            continue;
        int value = 0;
        if (cudaMemcpyAsync(&value, word, sizeof(int), cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
            cudaStreamSynchronize(stream) != cudaSuccess) {
            cudaGetLastError();
            return ATTN_ERR_CUDA;
        }
        if (value != 0) {
            const int zero = 0;
            if (cudaMemcpyAsync(word, &zero, sizeof(int), cudaMemcpyHostToDevice, stream) != cudaSuccess ||
                cudaStreamSynchronize(stream) != cudaSuccess) {
                cudaGetLastError();
                return ATTN_ERR_CUDA;
            }
            timed_out = true;
        }
    }
    return timed_out ? ATTN_ERR_DEVICE_TIMEOUT : ATTN_OK;
}

namespace {

// Shared by attn_decode_paged and attn_decode_paged_fp8 (k_scale, v_scale non-null for the latter).
int decode_paged_impl(const void *q, const void *k_pages, const void *v_pages, const float *k_scale,
                      const float *v_scale, const int *block_table, const int *seq_lens, void *o, float *lse, int B,
                      int Hq, int Hkv, int num_pages, int page_size, int pages_per_seq, int max_seq_len, float scale,
                      int decode_ctas, void *stream_ptr, bool fp8)
{
    using namespace attn_b200;
    if (!q || !k_pages || !v_pages || !block_table || !seq_lens || !o || !lse || (fp8 && (!k_scale || !v_scale)))
        return ATTN_ERR_NULL;
    if (B < 1 || B > kPagedMaxBatch || Hq < 1 || Hkv < 1 || num_pages < 1 || pages_per_seq < 1 || max_seq_len < 0 ||
        decode_ctas < 0)
        return ATTN_ERR_SHAPE;
    const bool page_ok = page_size == 16 || page_size == 32 || page_size == 64 ||
                         (page_size >= 128 && page_size % 128 == 0);
    if (!page_ok)
        return ATTN_ERR_SHAPE;
    if (Hq % Hkv != 0)
        return ATTN_ERR_GQA;
    // Page coordinates (page * Hkv + h), block-table offsets and output rows must fit in 32 bits.
    if (static_cast<long long>(num_pages) * Hkv > INT_MAX || static_cast<long long>(B) * pages_per_seq > INT_MAX ||
        static_cast<long long>(pages_per_seq) * page_size > INT_MAX || static_cast<long long>(B) * Hq > INT_MAX)
        return ATTN_ERR_SHAPE;
    if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(o) || !aligned16(lse) ||
        (reinterpret_cast<uintptr_t>(block_table) & 3u) || (reinterpret_cast<uintptr_t>(seq_lens) & 3u) ||
        (fp8 && (!aligned16(k_scale) || !aligned16(v_scale))))
        return ATTN_ERR_ALIGN;
    if (!(scale > 0.f) || !std::isfinite(scale))
        return ATTN_ERR_SCALE;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
    std::lock_guard<std::mutex> lock(g_mutex);
    int err = ATTN_OK;
    DeviceState *s = device_state(&err);
    if (!s)
        return err;
    DecodePlan plan;
    if (decode_plan_paged(B, Hq, Hkv, max_seq_len, decode_ctas, s->sm_count, &plan, fp8) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_SHAPE;
    }
    int rc = ensure_workspace(*s, static_cast<size_t>(plan.pairs), plan.partial_floats, stream);
    if (rc != ATTN_OK)
        return rc;
    DecodeArgs a;
    a.q = q;
    a.k = k_pages;
    a.v = v_pages;
    a.o = o;
    a.lse = lse;
    a.B = B;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.Skv = 0;
    a.D = 128;
    a.scale = scale;
    a.plan = plan;
    a.ws = s->partials;
    a.counters = s->counters;
    a.status = s->status;
    a.seq_lens = seq_lens;
    a.block_table = block_table;
    a.num_pages = num_pages;
    a.page_size = page_size;
    a.pages_per_seq = pages_per_seq;
    a.max_seq_len = max_seq_len;
    a.fp8 = fp8;
    a.k_scale = k_scale;
    a.v_scale = v_scale;
    if (launch_decode_tc(a, stream) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_LAUNCH;
    }
    return ATTN_OK;
}

}  // namespace

extern "C" int attn_prefill_paged(const void *q, const void *k_pages, const void *v_pages, const int *block_table,
                                  const int *seq_lens, void *o, float *lse, int B, int Hq, int Hkv, int Sq, int num_pages,
                                  int page_size, int pages_per_seq, int max_seq_len, float scale, int causal,
                                  void *stream_ptr)
{
    using namespace attn_b200;
    if (!q || !k_pages || !v_pages || !block_table || !seq_lens || !o || !lse)
        return ATTN_ERR_NULL;
    if (B < 1 || Hq < 1 || Hkv < 1 || Sq < 1 || num_pages < 1 || pages_per_seq < 1 || max_seq_len < 0)
        return ATTN_ERR_SHAPE;
    if (causal != 0 && causal != 1)
        return ATTN_ERR_SHAPE;
    const bool page_ok = page_size == 16 || page_size == 32 || page_size == 64 ||
                         (page_size >= 128 && page_size % 128 == 0);
    if (!page_ok)
        return ATTN_ERR_SHAPE;
    if (Hq % Hkv != 0)
        return ATTN_ERR_GQA;
    // Rows (b*Hq + h)*Sq + i, block-table offsets and key positions must fit in 32 bits.
    if (static_cast<long long>(B) * Hq * Sq > INT_MAX || static_cast<long long>(B) * pages_per_seq > INT_MAX ||
        static_cast<long long>(pages_per_seq) * page_size > INT_MAX)
        return ATTN_ERR_SHAPE;
    if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(o) || !aligned16(lse) ||
        (reinterpret_cast<uintptr_t>(block_table) & 3u) || (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
        return ATTN_ERR_ALIGN;
    if (!(scale > 0.f) || !std::isfinite(scale))
        return ATTN_ERR_SCALE;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
    std::lock_guard<std::mutex> lock(g_mutex);
    int err = ATTN_OK;
    DeviceState *s = device_state(&err);
    if (!s)
        return err;
    int rc = ensure_workspace(*s, 0, 0, stream);  // the status word
    if (rc != ATTN_OK)
        return rc;
    const int D = 128;
    PrefillArgs a;
    a.q = q;
    a.k = k_pages;
    a.v = v_pages;
    a.o = o;
    a.lse = lse;
    a.B = B;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.Sq = Sq;
    a.Skv = 0;
    a.D = D;
    a.scale = scale;
    a.causal = causal;
    a.status = s->status;
    a.sm_count = s->sm_count;
    a.qs = a.os = TensorStrides{static_cast<long long>(Hq) * Sq * D, static_cast<long long>(Sq) * D, D};
    a.ks = a.vs = TensorStrides{0, 0, 0};  // unused: the pages have their own layout
    a.seq_lens = seq_lens;
    a.block_table = block_table;
    a.num_pages = num_pages;
    a.page_size = page_size;
    a.pages_per_seq = pages_per_seq;
    a.max_seq_len = max_seq_len;
    int encode_error = 0;
    if (launch_prefill(a, stream, &encode_error) != cudaSuccess) {
        cudaGetLastError();
        return encode_error ? ATTN_ERR_CUDA : ATTN_ERR_LAUNCH;
    }
    return ATTN_OK;
}

extern "C" int attn_decode_paged(const void *q, const void *k_pages, const void *v_pages, const int *block_table,
                                 const int *seq_lens, void *o, float *lse, int B, int Hq, int Hkv, int num_pages,
                                 int page_size, int pages_per_seq, int max_seq_len, float scale, int decode_ctas,
                                 void *stream_ptr)
{
    return decode_paged_impl(q, k_pages, v_pages, nullptr, nullptr, block_table, seq_lens, o, lse, B, Hq, Hkv,
                             num_pages, page_size, pages_per_seq, max_seq_len, scale, decode_ctas, stream_ptr, false);
}

extern "C" int attn_decode_paged_fp8(const void *q, const void *k_pages, const void *v_pages, const float *k_scale,
                                     const float *v_scale, const int *block_table, const int *seq_lens, void *o,
                                     float *lse, int B, int Hq, int Hkv, int num_pages, int page_size,
                                     int pages_per_seq, int max_seq_len, float scale, int decode_ctas,
                                     void *stream_ptr)
{
    return decode_paged_impl(q, k_pages, v_pages, k_scale, v_scale, block_table, seq_lens, o, lse, B, Hq, Hkv,
                             num_pages, page_size, pages_per_seq, max_seq_len, scale, decode_ctas, stream_ptr, true);
}

extern "C" int attn_prefill_fp8(const void *q, const void *k8, const void *v8, const float *k_scale,
                                const float *v_scale, void *o, float *lse, int B, int Hq, int Hkv, int Sq, int Skv,
                                int D, float scale, int causal, void *stream_ptr)
{
    using namespace attn_b200;
    if (!q || !k8 || !v8 || !k_scale || !v_scale || !o || !lse)
        return ATTN_ERR_NULL;
    if (B < 1 || Hq < 1 || Hkv < 1 || Sq < 1 || Skv < 1 || (causal != 0 && causal != 1))
        return ATTN_ERR_SHAPE;
    if (Hq % Hkv != 0)
        return ATTN_ERR_GQA;
    if (D != 128)
        return ATTN_ERR_HEADDIM;
    // Flat row indices and tensor-map coordinates must fit in 32 bits; so must the grid.
    if (static_cast<long long>(B) * Hq * Sq > INT_MAX || static_cast<long long>(B) * Hkv * Skv > INT_MAX)
        return ATTN_ERR_SHAPE;
    if (causal && Sq > Skv)
        return ATTN_ERR_CAUSAL_SQ_GT_SKV;
    if (!aligned16(q) || !aligned16(k8) || !aligned16(v8) || !aligned16(k_scale) || !aligned16(v_scale) ||
        !aligned16(o) || !aligned16(lse))
        return ATTN_ERR_ALIGN;
    if (!(scale > 0.f) || !std::isfinite(scale))
        return ATTN_ERR_SCALE;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
    std::lock_guard<std::mutex> lock(g_mutex);
    int err = ATTN_OK;
    DeviceState *s = device_state(&err);
    if (!s)
        return err;
    int rc = ensure_workspace(*s, 0, 0, stream);  // the status word
    if (rc != ATTN_OK)
        return rc;
    PrefillFp8Args a;
    a.q = q;
    a.k8 = k8;
    a.v8 = v8;
    a.k_scale = k_scale;
    a.v_scale = v_scale;
    a.o = o;
    a.lse = lse;
    a.B = B;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.Sq = Sq;
    a.Skv = Skv;
    a.D = D;
    a.scale = scale;
    a.causal = causal;
    a.status = s->status;
    int encode_error = 0;
    const cudaError_t e = launch_prefill_fp8(a, stream, &encode_error);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return encode_error != 0 ? ATTN_ERR_CUDA : ATTN_ERR_LAUNCH;
    }
    return ATTN_OK;
}

extern "C" int attn_decode_fp8(const void *q, const void *k8, const void *v8, const float *k_scale,
                               const float *v_scale, void *o, float *lse, int B, int Hq, int Hkv, int Skv, int D,
                               float scale, int decode_ctas, void *stream_ptr)
{
    using namespace attn_b200;
    if (!q || !k8 || !v8 || !k_scale || !v_scale || !o || !lse)
        return ATTN_ERR_NULL;
    if (B < 1 || Hq < 1 || Hkv < 1 || Skv < 1 || decode_ctas < 0)
        return ATTN_ERR_SHAPE;
    if (Hq % Hkv != 0)
        return ATTN_ERR_GQA;
    if (D != 128)
        return ATTN_ERR_HEADDIM;
    // Tensor-map coordinates (rows of a kv head, b * Hkv + h) and output rows must fit in 32 bits.
    if (static_cast<long long>(B) * Hkv > INT_MAX || static_cast<long long>(B) * Hq > INT_MAX)
        return ATTN_ERR_SHAPE;
    if (!aligned16(q) || !aligned16(k8) || !aligned16(v8) || !aligned16(k_scale) || !aligned16(v_scale) ||
        !aligned16(o) || !aligned16(lse))
        return ATTN_ERR_ALIGN;
    if (!(scale > 0.f) || !std::isfinite(scale))
        return ATTN_ERR_SCALE;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
    std::lock_guard<std::mutex> lock(g_mutex);
    int err = ATTN_OK;
    DeviceState *s = device_state(&err);
    if (!s)
        return err;
    DecodePlan plan;
    if (decode_plan(B, Hq, Hkv, Skv, D, decode_ctas, s->sm_count, &plan, true) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_SHAPE;
    }
    int rc = ensure_workspace(*s, static_cast<size_t>(plan.pairs), plan.partial_floats, stream);
    if (rc != ATTN_OK)
        return rc;
    DecodeArgs a;
    a.q = q;
    a.k = k8;
    a.v = v8;
    a.o = o;
    a.lse = lse;
    a.B = B;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.Skv = Skv;
    a.D = D;
    a.scale = scale;
    a.plan = plan;
    a.ws = s->partials;
    a.counters = s->counters;
    a.status = s->status;
    a.fp8 = true;
    a.k_scale = k_scale;
    a.v_scale = v_scale;
    if (launch_decode_tc(a, stream) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_LAUNCH;
    }
    return ATTN_OK;
}

extern "C" int attn_lse_merge(float *o_acc, float *lse_acc, const void *o_part, const float *lse_part, void *o_out,
                              long long rows, int D, void *stream_ptr)
{
    using namespace attn_b200;
    if (!o_acc || !lse_acc || !o_part || !lse_part)
        return ATTN_ERR_NULL;
    if (rows < 0 || rows > (1LL << 40))
        return ATTN_ERR_SHAPE;
    if (D != 32 && D != 64 && D != 128)
        return ATTN_ERR_HEADDIM;
    if (!aligned16(o_acc) || !aligned16(o_part) || !aligned16(lse_acc) || !aligned16(lse_part) ||
        (o_out && !aligned16(o_out)))
        return ATTN_ERR_ALIGN;
    if (rows == 0)
        return ATTN_OK;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
    int err = ATTN_OK;
    DeviceState *s = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        s = device_state(&err);
    }
    if (!s)
        return err;
    if (launch_lse_merge(o_acc, lse_acc, o_part, lse_part, o_out, rows, D, s->sm_count, stream) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_LAUNCH;
    }
    return ATTN_OK;
}

extern "C" int attn_bwd(const void *q, const void *k, const void *v, const void *o, const void *dout, const float *lse,
                        void *dq, void *dk, void *dv, int B, int Hq, int Hkv, int Sq, int Skv, int D, float scale,
                        int causal, void *stream_ptr)
{
    using namespace attn_b200;
    int rc = validate(q, k, v, o, lse, B, Hq, Hkv, Sq, Skv, D, scale, causal);
    if (rc != ATTN_OK)
        return rc;
    if (!dout || !dq || !dk || !dv)
        return ATTN_ERR_NULL;
    if (!aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
        return ATTN_ERR_ALIGN;
    if (D != 128)
        return ATTN_ERR_HEADDIM;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
    std::lock_guard<std::mutex> lock(g_mutex);
    int err = ATTN_OK;
    DeviceState *s = device_state(&err);
    if (!s)
        return err;
    rc = ensure_workspace(*s, 0, 0, stream);  // the status word
    if (rc != ATTN_OK)
        return rc;
    const size_t need = bwd_workspace_bytes(B, Hq, Sq, D);
    if (s->bwd_bytes < need) {
        // Stream-ordered, as for the forward workspace: the old block is released on `stream` after
        // the work queued on it; nothing waits on the host.
        void *block = nullptr;
        if (cudaMallocAsync(&block, need, stream) != cudaSuccess) {
            cudaGetLastError();
            return ATTN_ERR_WORKSPACE;
        }
        if (s->bwd_block && cudaFreeAsync(s->bwd_block, stream) != cudaSuccess)
            cudaGetLastError();
        s->bwd_block = block;
        s->bwd_bytes = need;
    }
    BwdArgs a;
    a.q = q;
    a.k = k;
    a.v = v;
    a.o = o;
    a.dout = dout;
    a.lse = lse;
    a.dq = dq;
    a.dk = dk;
    a.dv = dv;
    a.B = B;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.Sq = Sq;
    a.Skv = Skv;
    a.D = D;
    a.scale = scale;
    a.causal = causal;
    a.ws = s->bwd_block;
    a.status = s->status;
    a.sm_count = s->sm_count;
    int encode_error = 0;
    if (launch_bwd(a, stream, &encode_error) != cudaSuccess) {
        cudaGetLastError();
        return encode_error ? ATTN_ERR_CUDA : ATTN_ERR_LAUNCH;
    }
    return ATTN_OK;
}

