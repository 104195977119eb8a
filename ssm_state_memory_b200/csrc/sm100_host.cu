// Host helpers shared by the tcgen05 kernels: TMA tensor maps (through the driver
// entry point, so the library does not link libcuda) and the SM count.
#include <cuda.h>

#include <cstdio>

#include "dart_internal.cuh"

namespace dart {

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q);
        if (e == cudaSuccess && q == cudaDriverEntryPointSuccess && ptr)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
        else
            set_last_error("cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)",
                           e == cudaSuccess ? cudaErrorSymbolNotFound : e);
    }
    return fn;
}

}  // namespace

bool make_tma_map_bf16(void *map, const void *base, uint64_t cols, uint64_t rows, uint64_t row_bytes,
                       uint32_t box_cols, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(static_cast<CUtensorMap *>(map), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base),
                    dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        char msg[192];
        snprintf(msg, sizeof(msg), "cuTensorMapEncodeTiled returned %d (cols %llu rows %llu stride %llu box %ux%u)",
                 (int)r, (unsigned long long)cols, (unsigned long long)rows, (unsigned long long)row_bytes, box_cols,
                 box_rows);
        set_last_error(msg, cudaErrorInvalidValue);
    }
    return r == CUDA_SUCCESS;
}

bool make_tma_map_f32_3d(void *map, const void *base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t stride1_bytes,
                         uint64_t stride2_bytes, uint32_t box0, uint32_t box1) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
    cuuint32_t box[3] = {box0, box1, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(static_cast<CUtensorMap *>(map), CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void *>(base),
                    dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        char msg[192];
        snprintf(msg, sizeof(msg), "cuTensorMapEncodeTiled returned %d (f32 3d %llu x %llu x %llu box %ux%u)", (int)r,
                 (unsigned long long)d0, (unsigned long long)d1, (unsigned long long)d2, box0, box1);
        set_last_error(msg, cudaErrorInvalidValue);
    }
    return r == CUDA_SUCCESS;
}

bool make_tma_map_bf16_3d(void *map, const void *base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t stride1_bytes,
                          uint64_t stride2_bytes, uint32_t box0, uint32_t box1) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
    cuuint32_t box[3] = {box0, box1, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(static_cast<CUtensorMap *>(map), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base),
                    dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        char msg[192];
        snprintf(msg, sizeof(msg), "cuTensorMapEncodeTiled returned %d (bf16 3d %llu x %llu x %llu box %ux%u)", (int)r,
                 (unsigned long long)d0, (unsigned long long)d1, (unsigned long long)d2, box0, box1);
        set_last_error(msg, cudaErrorInvalidValue);
    }
    return r == CUDA_SUCCESS;
}

static int current_device() {
    int dev = 0;
    cudaGetDevice(&dev);
    return dev;
}

bool device_flag_set(unsigned long long flags) {
    const int dev = current_device();
    return dev >= 0 && dev < 64 && ((flags >> dev) & 1ull);
}

void set_device_flag(unsigned long long *flags) {
    const int dev = current_device();
    if (dev >= 0 && dev < 64) *flags |= 1ull << dev;
}

int device_sm_count() {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

}  // namespace dart
