// dart_sma_decode_noalloc: single-token decode whose scratch lives in a fixed
// device array owned by the library, for callers that cannot allocate.
//
// Who needs this: code that is handed only its input and output buffers and may
// not allocate device memory itself, for example a plug-in running inside a
// serving framework that owns every device allocation and forbids cudaMalloc on
// its request threads (an allocation can synchronise the device and can fail
// under memory pressure in the middle of a request). dart_sma_decode needs a
// caller-provided workspace for its per-split partial results; this variant
// keeps them in `g_decode_scratch` below instead.
//
// The scratch array is a file-scope __device__ array: every GPU that loads the
// library holds these kMaxScratchBytes until the process exits, and every call
// on a device uses the same array. Each call writes every partial it later
// reads, so nothing in the array has to start at zero and stale contents from
// an earlier call are never used. Calls whose kernels overlap on the GPU (two
// streams, or two host threads) race on the array and must be serialised by the
// caller.
#include <mutex>

#include "dart_internal.cuh"

namespace dart {
namespace {

constexpr size_t kMaxScratchBytes = size_t(4) << 20;  // 4 MiB of fp32 partials per device

static __device__ __align__(256) unsigned char g_decode_scratch[kMaxScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once per
// device (with that device current) on the first call and kept for the life of
// the process: after cudaDeviceReset the kept address would be stale, so the
// entry point must not be used on a device after its context was reset. The
// host-side symbol `g_decode_scratch` is only a stand-in for the device array and
// must never be passed to a kernel directly.
cudaError_t scratch_address(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_setup_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace
}  // namespace dart

using namespace dart;

extern "C" dart_status dart_sma_decode_noalloc(int64_t batch, int64_t nheads, int64_t ngroups, int64_t dstate,
                                               int64_t headdim, int64_t n_chunks, int64_t chunk_stride,
                                               dart_dtype dtype, const void *Q, const void *C, const void *E,
                                               const void *Y, const float *g, int64_t g_sb, int64_t g_sh,
                                               const void *cache, void *out, float *lse, void *stream) {
    // same size rules as dart_sma_decode (an unsupported shape has no workspace size)
    const size_t need = dart_decode_workspace_size(batch, nheads, dstate, headdim, n_chunks, dtype);
    if (dtype != DART_F32 && dtype != DART_BF16) return DART_ERR_DTYPE;
    if (batch <= 0 || nheads <= 0 || ngroups <= 0 || dstate <= 0 || headdim <= 0 || n_chunks < 0 ||
        chunk_stride < n_chunks || chunk_stride <= 0 || nheads % ngroups != 0)
        return DART_ERR_DIMS;
    if (need == 0) return DART_ERR_UNSUPPORTED;
    if (need > kMaxScratchBytes) return DART_ERR_WORKSPACE;  // partials would not fit the fixed array
    if (!Q || !C || !E || !Y || !g || !cache || !out) return DART_ERR_NULL;
    if (!aligned16(Q) || !aligned16(C) || !aligned16(E) || !aligned16(Y) || !aligned16(cache) || !aligned16(out) ||
        (lse && !aligned16(lse)) || (reinterpret_cast<uintptr_t>(g) & 3))
        return DART_ERR_ALIGN;
    if (g_sb < 0 || g_sh < 0) return DART_ERR_DIMS;
    void *scratch = nullptr;
    cudaError_t e = scratch_address(&scratch);
    if (e != cudaSuccess) {
        set_last_error("cudaGetSymbolAddress(decode scratch)", e);
        return DART_ERR_CUDA;
    }
    DecodeArgs a{};
    a.Bt = batch;
    a.H = nheads;
    a.G = ngroups;
    a.N = dstate;
    a.P = headdim;
    a.n_chunks = n_chunks;
    a.chunk_stride = chunk_stride;
    a.Q = Q;
    a.C = C;
    a.E = E;
    a.Y = Y;
    a.g = g;
    a.g_sb = g_sb;
    a.g_sh = g_sh;
    a.cache = cache;
    a.out = out;
    a.lse = lse;
    a.partials = static_cast<float *>(scratch);
    a.splits = decode_splits(batch, nheads, n_chunks);
    e = launch_sma_decode(a, dtype == DART_BF16, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? DART_OK : DART_ERR_CUDA;
}
