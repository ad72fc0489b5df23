// forward_noalloc.cu -- bitnet_hbitlinear_forward_noalloc: the H-BitLinear forward
// for callers that cannot allocate device memory.
//
// bitnet_hbitlinear_forward keeps the int8 activation codes and per-token scales
// between its two kernels in a workspace the caller allocates.  Some callers have
// no way to do that: a plugin or extension interface that hands a kernel only its
// input and output buffers, a runtime that owns all device memory in a
// preplanned arena, or a latency-critical path that must never reach cudaMalloc
// (which can synchronise the device).  This entry point serves them: the scratch
// lives in a fixed-size array in the library's own device memory instead.
//
// The array is a file-scope __device__ variable, so every GPU that loads the
// library holds it (kNoAllocScratchBytes) until the process exits.  Its host-side
// name is only a stand-in for the device symbol; the kernels receive the device
// address obtained from cudaGetSymbolAddress, looked up once per device and kept in
// an atomic per-device cache (two host threads making their first call on a device at
// once both look it up and store the same address).  cudaDeviceReset destroys the
// module's device memory: after one, the cached address is stale, so a process that
// resets a device must not call this entry point on it again.
#include <atomic>

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "host.h"

namespace bitnet {

namespace {

constexpr size_t kNoAllocScratchBytes = BITNET_NOALLOC_SCRATCH_BYTES;

// Shared by every call on a device; holds the last call's codes and scales.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

std::atomic<uint8_t *> g_scratch_addr[kMaxDevices];

size_t round256(size_t v) { return (v + 255) & ~(size_t)255; }

// Device address of this device's scratch array (set up on first use per device,
// with that device current).
cudaError_t scratch_address(uint8_t **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    uint8_t *p = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (!p) {
        e = cudaGetSymbolAddress((void **)&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev].store(p, std::memory_order_release);
    }
    *out = p;
    return cudaSuccess;
}

}  // namespace

}  // namespace bitnet

using namespace bitnet;

extern "C" bitnet_status_t bitnet_hbitlinear_forward_noalloc(const void *X, bitnet_dtype_t xdt, int64_t M,
                                                              int64_t K, const float *gain, float eps, int fwht,
                                                              bitnet_act_mode_t mode, const uint8_t *packed,
                                                              const float *alpha, int64_t N, float *out,
                                                              void *stream) {
    // The argument rules of bitnet_hbitlinear_forward, from the same validator.
    const bitnet_status_t st = validate_forward(X, xdt, M, K, gain, fwht, mode, packed, alpha, N, out);
    if (st != BITNET_OK || M == 0) return st;
    // Codes [M][K], scales [M] (each 256-byte aligned) and the split-K tile counters
    // must fit the fixed array.
    const size_t codes_bytes = round256((size_t)M * (size_t)K);
    const size_t scales_bytes = round256((size_t)M * sizeof(float));
    const size_t need = codes_bytes + scales_bytes + (size_t)kSplitCounters * sizeof(int);
    if (need > kNoAllocScratchBytes) return BITNET_ERR_WORKSPACE;

    uint8_t *scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return BITNET_ERR_CUDA;
    int8_t *codes = reinterpret_cast<int8_t *>(scratch);
    float *scale_x = reinterpret_cast<float *>(scratch + codes_bytes);
    int *tile_cnt = reinterpret_cast<int *>(scratch + codes_bytes + scales_bytes);
    // Nothing in the array needs clearing beforehand: the forward's first kernel writes
    // every code and scale that is read afterwards (the decode kernel that runs the
    // activation step itself writes them for the record only), and act_quant zeroes
    // the counters when the GEMM splits K.
    const cudaError_t e = forward_kernels(X, xdt, M, K, gain, eps, fwht, mode, packed, alpha, N, out, codes, scale_x,
                                          tile_cnt, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? BITNET_OK : BITNET_ERR_CUDA;
}
