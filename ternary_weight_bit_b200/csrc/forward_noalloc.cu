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
// address obtained from cudaGetSymbolAddress, looked up once per device.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "host.h"

namespace bitnet {

namespace {

constexpr size_t kNoAllocScratchBytes = BITNET_NOALLOC_SCRATCH_BYTES;

// Shared by every call on a device; holds the last call's codes and scales.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

uint8_t *g_scratch_addr[kMaxDevices] = {};

size_t round256(size_t v) { return (v + 255) & ~(size_t)255; }

// Device address of this device's scratch array (set up on first use per device).
cudaError_t scratch_address(uint8_t **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (!g_scratch_addr[dev]) {
        uint8_t *p = nullptr;
        e = cudaGetSymbolAddress((void **)&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

}  // namespace bitnet

using namespace bitnet;

extern "C" bitnet_status_t bitnet_hbitlinear_forward_noalloc(const void *X, bitnet_dtype_t xdt, int64_t M,
                                                              int64_t K, const float *gain, float eps, int fwht,
                                                              bitnet_act_mode_t mode, const uint8_t *packed,
                                                              const float *alpha, int64_t N, float *out,
                                                              void *stream) {
    // Argument rules are those of bitnet_hbitlinear_forward.
    if (xdt != BITNET_F32 && xdt != BITNET_BF16) return BITNET_ERR_INVALID_ARG;
    if (mode != BITNET_ACT_INT8_ABSMAX && mode != BITNET_ACT_INT4_ABSMEAN) return BITNET_ERR_INVALID_ARG;
    if (fwht != 0 && fwht != 1) return BITNET_ERR_INVALID_ARG;
    if (M < 0 || N < 1 || M > ((int64_t)1 << 30) || N > ((int64_t)1 << 30)) return BITNET_ERR_INVALID_ARG;
    if (K <= 0 || K % 128 != 0 || K > 32768) return BITNET_ERR_UNSUPPORTED_SHAPE;
    if (fwht && (K & (K - 1)) != 0) return BITNET_ERR_NOT_POW2;
    if (M == 0) return BITNET_OK;
    if (!X || !packed || !alpha || !out) return BITNET_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(packed) || !aligned16(alpha) || !aligned16(out) || (gain && !aligned16(gain)))
        return BITNET_ERR_INVALID_ARG;
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
    // Nothing in the array needs clearing beforehand: act_quant writes every code and
    // scale the GEMM reads, and zeroes the counters when the GEMM splits K.
    const cudaError_t e = forward_kernels(X, xdt, M, K, gain, eps, fwht, mode, packed, alpha, N, out, codes, scale_x,
                                          tile_cnt, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? BITNET_OK : BITNET_ERR_CUDA;
}
