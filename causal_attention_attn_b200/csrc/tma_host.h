/*
 * tma_host.h — host-side construction of TMA tensor maps over the library's tensors.
 *
 * The driver's cuTensorMapEncodeTiled is reached through cudaGetDriverEntryPoint, so the library
 * does not link against libcuda. Internal to the library; not part of the public ABI.
 */
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <mutex>

namespace attn_b200 {

// The driver's tensor-map encoder, looked up once; null when the driver does not provide it.
inline PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn()
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

// 3-D map over a contiguous bf16 tensor [BH][S][D] with a box of (box_inner elements of D,
// box_rows rows of S, 1). Reads outside the tensor fill with zeros. Returns false (and the driver's
// code in *err) when the driver rejects the map: base not 16-byte aligned, a stride not a multiple
// of 16 bytes, or a box the swizzle mode cannot hold.
inline bool make_map(PFN_cuTensorMapEncodeTiled_v12000 encode, CUtensorMap *map, const void *base, int D, int S,
                     int BH, int box_inner, int box_rows, CUtensorMapSwizzle swizzle, int *err)
{
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(S), static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(S) * D * 2};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_rows), 1u};
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

// As make_map for a contiguous fp32 tensor [BH][S][D] (the target of tiled reduce-adds).
inline bool make_map_f32(PFN_cuTensorMapEncodeTiled_v12000 encode, CUtensorMap *map, void *base, int D, int S, int BH,
                         int box_inner, int box_rows, CUtensorMapSwizzle swizzle, int *err)
{
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(S), static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 4, static_cast<cuuint64_t>(S) * D * 4};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_rows), 1u};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        *err = static_cast<int>(r);
        return false;
    }
    return true;
}

// As make_map for a contiguous tensor of 8-bit elements [BH][S][D] (D bytes per row), with a box
// of (box_inner bytes, box_rows rows, 1).
inline bool make_map_u8(PFN_cuTensorMapEncodeTiled_v12000 encode, CUtensorMap *map, const void *base, int D, int S,
                        int BH, int box_inner, int box_rows, CUtensorMapSwizzle swizzle, int *err)
{
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(S), static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(S) * D};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_rows), 1u};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        *err = static_cast<int>(r);
        return false;
    }
    return true;
}

// Element strides of a [batch][head][row][dim] tensor whose dim is contiguous: the layout of q, k,
// v or o. Heads-major contiguous is (H*S*D, S*D, D); token-major [B, S, H, D] is (S*H*D, D, H*D).
struct Strides {
    long long b, h, s;
};

inline Strides contiguous_strides(int H, int S, int D)
{
    return Strides{static_cast<long long>(H) * S * D, static_cast<long long>(S) * D, static_cast<long long>(D)};
}

// 4-D map (dim, row, head, batch) over a tensor with element strides `st` and `elem_bytes`-byte
// elements (2: bf16, 1: e4m3 codes), box (box_inner, box_rows, 1, 1). Reads outside the tensor fill
// with zeros. Returns false (and the driver's code in *err) when the driver rejects the map (a
// stride not a multiple of 16 bytes, an unaligned base, a box the swizzle mode cannot hold).
inline bool make_map4(PFN_cuTensorMapEncodeTiled_v12000 encode, CUtensorMap *map, const void *base, int elem_bytes,
                      int D, int S, int H, int B, Strides st, int box_inner, int box_rows, CUtensorMapSwizzle swizzle,
                      int *err)
{
    cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(S), static_cast<cuuint64_t>(H),
                          static_cast<cuuint64_t>(B)};
    cuuint64_t strides[3] = {static_cast<cuuint64_t>(st.s) * elem_bytes, static_cast<cuuint64_t>(st.h) * elem_bytes,
                             static_cast<cuuint64_t>(st.b) * elem_bytes};
    cuuint32_t box[4] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_rows), 1u, 1u};
    cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    CUresult r = encode(map, elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 4,
                        const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        *err = static_cast<int>(r);
        return false;
    }
    return true;
}

}  // namespace attn_b200
