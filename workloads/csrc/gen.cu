// Device side of the workloads' counter-based generator (see workloads/__init__.py):
// SplitMix64 (Steele, Lea & Flood, OOPSLA 2014) of counter i under a stream key,
// summed over its four 16-bit fields as an Irwin-Hall(4) variate, scaled in fp32
// and rounded to bf16 (round to nearest even). Bit-identical to the numpy side.
// This generates inputs only; it holds none of the DART arithmetic.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

__device__ __forceinline__ uint64_t splitmix64(uint64_t key, uint64_t idx) {
    uint64_t z = key + (idx + 1ull) * 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

__global__ void k_fill_irwin_hall_bf16(__nv_bfloat16 *dst, int64_t count, uint64_t key, uint64_t start, float scale) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < count; i += (int64_t)gridDim.x * blockDim.x) {
        uint64_t z = splitmix64(key, start + (uint64_t)i);
        int32_t s = (int32_t)(z & 0xffff) + (int32_t)((z >> 16) & 0xffff) + (int32_t)((z >> 32) & 0xffff) +
                    (int32_t)(z >> 48) - 131070;
        dst[i] = __float2bfloat16_rn(__fmul_rn((float)s, scale));
    }
}

}  // namespace

extern "C" int dartw_fill_irwin_hall_bf16(void *dst, int64_t count, uint64_t key, uint64_t start, float scale,
                                          void *stream) {
    if (!dst || count < 0) return 1;
    if (count == 0) return 0;
    int64_t blocks = (count + 255) / 256;
    if (blocks > 148 * 32) blocks = 148 * 32;
    k_fill_irwin_hall_bf16<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<__nv_bfloat16 *>(dst), count, key, start, scale);
    return cudaGetLastError() == cudaSuccess ? 0 : 2;
}
