// bitnet_abi.cu -- the C ABI of libbitnet.so (declared in include/bitnet.h):
// argument validation, TMA descriptor encoding, kernel selection and launch.
// Nothing here allocates device memory; every launch goes to the caller's stream.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "host.h"

namespace bitnet {

// The device status word (one per device that loads the library).
static __device__ int g_device_status = 0;

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bitnet_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? BITNET_OK : BITNET_ERR_CUDA; }

constexpr int64_t kMaxK = 32768;
constexpr int64_t kMaxRows = (int64_t)1 << 30;  // M and N bounds (TMA coordinates are int32)

bitnet_status_t check_k(int64_t K, int fwht) {
    if (K <= 0 || K % 128 != 0 || K > kMaxK) return BITNET_ERR_UNSUPPORTED_SHAPE;
    if (fwht && (K & (K - 1)) != 0) return BITNET_ERR_NOT_POW2;
    return BITNET_OK;
}

size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

}  // namespace

bool make_tmap_u8_2d(CUtensorMap *map, const void *base, uint64_t row_bytes, uint64_t rows, uint32_t box_x,
                     uint32_t box_y, CUtensorMapSwizzle swizzle) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {row_bytes, rows};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_x, box_y};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_out_2d(CUtensorMap *map, const void *base, bool bf16, uint64_t cols, uint64_t rows, uint32_t box_x,
                      uint32_t box_y) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * (bf16 ? 2 : 4)};
    const cuuint32_t box[2] = {box_x, box_y};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
              const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int *device_status_ptr() {
    static int *ptrs[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev >= kMaxDevices) return nullptr;
    if (!ptrs[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
        ptrs[dev] = static_cast<int *>(p);
    }
    return ptrs[dev];
}

int sm_count() {
    static int counts[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev >= kMaxDevices) return 148;
    if (!counts[dev]) {
        int c = 0;
        if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || c <= 0) c = 148;
        counts[dev] = c;
    }
    return counts[dev];
}

namespace {

__global__ void wait_selftest_kernel(uint64_t limit_ns, int *status) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(&bar, 0, status, limit_ns);  // nothing ever arrives
}

bitnet_status_t validate_gemm(const int8_t *codes, const float *scale_x, int mode, const uint8_t *packed,
                              const float *alpha, int64_t M, int64_t N, int64_t K, const void *out,
                              const int32_t *acc_out) {
    if (mode != BITNET_ACT_INT8_ABSMAX && mode != BITNET_ACT_INT4_ABSMEAN) return BITNET_ERR_INVALID_ARG;
    if (M < 0 || N < 1 || M > kMaxRows || N > kMaxRows) return BITNET_ERR_INVALID_ARG;
    bitnet_status_t st = check_k(K, 0);
    if (st != BITNET_OK) return st;
    if (M == 0) return BITNET_OK;
    if (!codes || !scale_x || !packed || !alpha || !out) return BITNET_ERR_INVALID_ARG;
    if (!aligned16(codes) || !aligned16(packed) || !aligned16(out) || !aligned16(scale_x) ||
        !aligned16(alpha) || (acc_out && !aligned16(acc_out)))
        return BITNET_ERR_INVALID_ARG;
    return BITNET_OK;
}

// Checks the activation-side inputs; codes/scale_x are checked only when check_outputs.
bitnet_status_t validate_act(const void *X, int xdt, int64_t M, int64_t K, const float *gain, int fwht, int mode,
                             const int8_t *codes, const float *scale_x, bool check_outputs) {
    if (xdt != BITNET_F32 && xdt != BITNET_BF16) return BITNET_ERR_INVALID_ARG;
    if (mode != BITNET_ACT_INT8_ABSMAX && mode != BITNET_ACT_INT4_ABSMEAN) return BITNET_ERR_INVALID_ARG;
    if (fwht != 0 && fwht != 1) return BITNET_ERR_INVALID_ARG;
    if (M < 0 || M > kMaxRows) return BITNET_ERR_INVALID_ARG;
    bitnet_status_t st = check_k(K, fwht);
    if (st != BITNET_OK) return st;
    if (M == 0) return BITNET_OK;
    if (!X || !aligned16(X) || (gain && !aligned16(gain))) return BITNET_ERR_INVALID_ARG;
    if (check_outputs && (!codes || !scale_x || !aligned16(codes) || !aligned16(scale_x)))
        return BITNET_ERR_INVALID_ARG;
    return BITNET_OK;
}

// The standalone GEMM.  With a workspace (tile_cnt, kSplitCounters ints) an fp32
// GEMM of few output tiles may split K as the forward does; the counters (and, for
// more than two splits, the output) are zeroed by memsets on the stream first.
cudaError_t run_gemm(const int8_t *codes, const float *scale_x, int mode, const uint8_t *packed,
                     const float *alpha, int64_t M, int64_t N, int64_t K, void *out, bool out_bf16,
                     int32_t *acc_out, bool pdl, cudaStream_t s, int *tile_cnt = nullptr) {
    if (M <= kGemvMaxM)
        return launch_gemv(codes, scale_x, mode, packed, alpha, (int)M, (int)N, (int)K, out, acc_out, pdl, s,
                           out_bf16);
    GemmPlan plan{0, 1};
    if (tile_cnt && !out_bf16) {
        plan = gemm_plan((int)M, (int)N, (int)K, sm_count(), kSplitCounters);
        if (plan.splits > 1) {
            cudaError_t e = cudaMemsetAsync(tile_cnt, 0, (size_t)kSplitCounters * sizeof(int), s);
            if (e == cudaSuccess && plan.splits > 2) e = cudaMemsetAsync(out, 0, (size_t)M * (size_t)N * 4, s);
            if (e != cudaSuccess) return e;
            pdl = false;  // the kernel follows a memset, not a kernel
        }
    }
    return launch_gemm_tc(codes, scale_x, mode, packed, alpha, (int)M, (int)N, (int)K, out, acc_out, pdl, s, plan,
                          plan.splits > 1 ? tile_cnt : nullptr, out_bf16);
}

}  // namespace

// act_quant into (codes, scale_x), then the GEMV or the tcgen05 GEMM, the second
// launched with programmatic dependent launch.  A GEMM whose output has few tiles splits K:
// act_quant then also zeroes `out` and the tile counters for it.
cudaError_t forward_kernels(const void *X, bitnet_dtype_t xdt, int64_t M, int64_t K, const float *gain, float eps,
                            int fwht, bitnet_act_mode_t mode, const uint8_t *packed, const float *alpha,
                            int64_t N, void *out, int8_t *codes, float *scale_x, int *tile_cnt, cudaStream_t s,
                            const void *up, bool out_bf16) {
    GemmPlan plan{0, 1};
    ZeroFill zf;
    if (M > kGemvMaxM) {
        // a bf16 output cannot hold the int32 sums of a split GEMM: never split it
        plan = gemm_plan((int)M, (int)N, (int)K, sm_count(), out_bf16 ? 0 : kSplitCounters);
        if (plan.splits == 2) {
            zf.cnt = tile_cnt;  // arrival counters and ready flags; the output needs no zeroing
            zf.cnt_n = kSplitCounters;
        } else if (plan.splits > 1) {
            zf.rows = reinterpret_cast<uint32_t *>(out);
            zf.row_words = (int)N;
            zf.cnt = tile_cnt;
            zf.cnt_n = (int)(((N + 127) / 128) * ((M + plan.token_tile - 1) / plan.token_tile));
        }
    }
    cudaError_t e = up ? launch_act_quant_swiglu(X, up, xdt == BITNET_BF16, M, (int)K, gain, eps, fwht, mode, codes,
                                                 scale_x, s, zf)
                       : launch_act_quant(X, xdt == BITNET_BF16, M, (int)K, gain, eps, fwht, mode, codes, scale_x, s, zf);
    if (e != cudaSuccess) return e;
    if (M <= kGemvMaxM)
        return launch_gemv(codes, scale_x, mode, packed, alpha, (int)M, (int)N, (int)K, out, nullptr, true, s,
                           out_bf16);
    return launch_gemm_tc(codes, scale_x, mode, packed, alpha, (int)M, (int)N, (int)K, out, nullptr, true, s, plan,
                          tile_cnt, out_bf16);
}

// Argument rules of every forward entry point (workspace excluded).
bitnet_status_t validate_forward(const void *X, bitnet_dtype_t xdt, int64_t M, int64_t K, const float *gain,
                                 int fwht, bitnet_act_mode_t mode, const uint8_t *packed, const float *alpha,
                                 int64_t N, const void *out) {
    if (N < 1 || N > kMaxRows) return BITNET_ERR_INVALID_ARG;
    bitnet_status_t st = validate_act(X, xdt, M, K, gain, fwht, mode, nullptr, nullptr, false);
    if (st != BITNET_OK || M == 0) return st;
    if (!packed || !alpha || !out || !aligned16(packed) || !aligned16(alpha) || !aligned16(out))
        return BITNET_ERR_INVALID_ARG;
    return BITNET_OK;
}

cudaError_t launch_wait_selftest(uint32_t limit_us, cudaStream_t s) {
    wait_selftest_kernel<<<1, 32, 0, s>>>((uint64_t)limit_us * 1000ull, device_status_ptr());
    return cudaGetLastError();
}

}  // namespace bitnet

using namespace bitnet;

extern "C" {

int bitnet_abi_version(void) { return BITNET_ABI_VERSION; }

const char *bitnet_status_string(bitnet_status_t s) {
    switch (s) {
        case BITNET_OK: return "ok";
        case BITNET_ERR_INVALID_ARG: return "invalid argument (null or misaligned pointer, bad enum or size)";
        case BITNET_ERR_UNSUPPORTED_SHAPE: return "unsupported shape (K must be a multiple of 128, at most 32768)";
        case BITNET_ERR_NOT_POW2: return "FWHT needs K to be a power of two";
        case BITNET_ERR_CUDA: return "CUDA runtime error";
        case BITNET_ERR_TIMEOUT: return "a kernel gave up on a bounded wait";
        case BITNET_ERR_WORKSPACE: return "workspace missing or too small";
        default: return "unknown status";
    }
}

size_t bitnet_pack_workspace_bytes(int64_t N, int64_t K) {
    (void)N;
    (void)K;
    return align256(pack_workspace_bytes());
}

bitnet_status_t bitnet_pack_ternary(const float *W, int64_t N, int64_t K, float eps, uint8_t *packed, float *alpha,
                                    void *ws, size_t ws_bytes, void *stream) {
    if (N < 1 || N > kMaxRows) return BITNET_ERR_INVALID_ARG;
    bitnet_status_t st = check_k(K, 0);
    if (st != BITNET_OK) return st;
    if (!W || !packed || !alpha) return BITNET_ERR_INVALID_ARG;
    if (!aligned16(W) || !aligned16(packed) || !aligned16(alpha)) return BITNET_ERR_INVALID_ARG;
    if (!ws || ws_bytes < bitnet_pack_workspace_bytes(N, K) || (reinterpret_cast<uintptr_t>(ws) & 255u))
        return BITNET_ERR_WORKSPACE;
    return from_cuda(launch_pack(W, N, K, eps, packed, alpha, ws, static_cast<cudaStream_t>(stream)));
}

bitnet_status_t bitnet_act_quant(const void *X, bitnet_dtype_t xdt, int64_t M, int64_t K, const float *gain,
                                 float eps, int fwht, bitnet_act_mode_t mode, int8_t *codes, float *scale_x,
                                 void *stream) {
    bitnet_status_t st = validate_act(X, xdt, M, K, gain, fwht, mode, codes, scale_x, true);
    if (st != BITNET_OK || M == 0) return st;
    return from_cuda(launch_act_quant(X, xdt == BITNET_BF16, M, (int)K, gain, eps, fwht, mode, codes, scale_x,
                                      static_cast<cudaStream_t>(stream)));
}

bitnet_status_t bitnet_ternary_gemm(const int8_t *codes, const float *scale_x, bitnet_act_mode_t mode,
                                    const uint8_t *packed, const float *alpha, int64_t M, int64_t N, int64_t K,
                                    float *out, int32_t *acc_out, void *ws, size_t ws_bytes, void *stream) {
    bitnet_status_t st = validate_gemm(codes, scale_x, mode, packed, alpha, M, N, K, out, acc_out);
    if (st != BITNET_OK || M == 0) return st;
    if (ws && (ws_bytes < bitnet_gemm_workspace_bytes(M, N, K) || (reinterpret_cast<uintptr_t>(ws) & 255u)))
        return BITNET_ERR_WORKSPACE;
    return from_cuda(run_gemm(codes, scale_x, mode, packed, alpha, M, N, K, out, false, acc_out, true,
                              static_cast<cudaStream_t>(stream), static_cast<int *>(ws)));
}

bitnet_status_t bitnet_ternary_gemm_ex(const int8_t *codes, const float *scale_x, bitnet_act_mode_t mode,
                                       const uint8_t *packed, const float *alpha, int64_t M, int64_t N, int64_t K,
                                       void *out, bitnet_dtype_t out_dt, int32_t *acc_out, void *stream) {
    if (out_dt != BITNET_F32 && out_dt != BITNET_BF16) return BITNET_ERR_INVALID_ARG;
    bitnet_status_t st = validate_gemm(codes, scale_x, mode, packed, alpha, M, N, K, out, acc_out);
    if (st != BITNET_OK || M == 0) return st;
    return from_cuda(run_gemm(codes, scale_x, mode, packed, alpha, M, N, K, out, out_dt == BITNET_BF16, acc_out,
                              true, static_cast<cudaStream_t>(stream)));
}

size_t bitnet_forward_workspace_bytes(int64_t M, int64_t K) {
    if (M <= 0 || K < 0) return 0;
    // codes [M][K], scales [M], then the split-K tile counters of the GEMM
    return align256((size_t)M * (size_t)K) + align256((size_t)M * sizeof(float)) +
           (size_t)kSplitCounters * sizeof(int);
}

size_t bitnet_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K) {
    (void)M;
    (void)N;
    (void)K;
    return (size_t)kSplitCounters * sizeof(int);  // tile counters and ready flags of a split K
}

size_t bitnet_workspace_bytes(int64_t M, int64_t N, int64_t K) {
    size_t need = bitnet_pack_workspace_bytes(N, K);
    const size_t f = bitnet_forward_workspace_bytes(M, K), g = bitnet_gemm_workspace_bytes(M, N, K);
    if (f > need) need = f;
    if (g > need) need = g;
    return need;
}


namespace {
bitnet_status_t forward_ws(const void *X, const void *up, bitnet_dtype_t xdt, int64_t M, int64_t K,
                           const float *gain, float eps, int fwht, bitnet_act_mode_t mode, const uint8_t *packed,
                           const float *alpha, int64_t N, void *out, bool out_bf16, void *ws, size_t ws_bytes,
                           void *stream) {
    bitnet_status_t st = validate_forward(X, xdt, M, K, gain, fwht, mode, packed, alpha, N, out);
    if (st != BITNET_OK || M == 0) return st;
    if (!ws || ws_bytes < bitnet_forward_workspace_bytes(M, K) || (reinterpret_cast<uintptr_t>(ws) & 255u))
        return BITNET_ERR_WORKSPACE;
    int8_t *codes = static_cast<int8_t *>(ws);
    float *scale_x = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + align256((size_t)M * (size_t)K));
    int *tile_cnt = reinterpret_cast<int *>(reinterpret_cast<uint8_t *>(scale_x) + align256((size_t)M * sizeof(float)));
    return from_cuda(forward_kernels(X, xdt, M, K, gain, eps, fwht, mode, packed, alpha, N, out, codes, scale_x,
                                     tile_cnt, static_cast<cudaStream_t>(stream), up, out_bf16));
}
}  // namespace

bitnet_status_t bitnet_hbitlinear_forward(const void *X, bitnet_dtype_t xdt, int64_t M, int64_t K,
                                          const float *gain, float eps, int fwht, bitnet_act_mode_t mode,
                                          const uint8_t *packed, const float *alpha, int64_t N, float *out,
                                          void *ws, size_t ws_bytes, void *stream) {
    return forward_ws(X, nullptr, xdt, M, K, gain, eps, fwht, mode, packed, alpha, N, out, false, ws, ws_bytes,
                      stream);
}

bitnet_status_t bitnet_hbitlinear_forward_ex(const void *X, bitnet_dtype_t xdt, int64_t M, int64_t K,
                                             const float *gain, float eps, int fwht, bitnet_act_mode_t mode,
                                             const uint8_t *packed, const float *alpha, int64_t N, void *out,
                                             bitnet_dtype_t out_dt, void *ws, size_t ws_bytes, void *stream) {
    if (out_dt != BITNET_F32 && out_dt != BITNET_BF16) return BITNET_ERR_INVALID_ARG;
    return forward_ws(X, nullptr, xdt, M, K, gain, eps, fwht, mode, packed, alpha, N, out, out_dt == BITNET_BF16,
                      ws, ws_bytes, stream);
}

bitnet_status_t bitnet_act_quant_swiglu(const void *gate, const void *up, bitnet_dtype_t xdt, int64_t M, int64_t K,
                                        const float *gain, float eps, int fwht, bitnet_act_mode_t mode, int8_t *codes,
                                        float *scale_x, void *stream) {
    bitnet_status_t st = validate_act(gate, xdt, M, K, gain, fwht, mode, codes, scale_x, true);
    if (st != BITNET_OK || M == 0) return st;
    if (!up || !aligned16(up)) return BITNET_ERR_INVALID_ARG;
    return from_cuda(launch_act_quant_swiglu(gate, up, xdt == BITNET_BF16, M, (int)K, gain, eps, fwht, mode, codes,
                                             scale_x, static_cast<cudaStream_t>(stream)));
}

bitnet_status_t bitnet_hbitlinear_forward_swiglu(const void *gate, const void *up, bitnet_dtype_t xdt, int64_t M,
                                                 int64_t K, const float *gain, float eps, int fwht,
                                                 bitnet_act_mode_t mode, const uint8_t *packed, const float *alpha,
                                                 int64_t N, float *out, void *ws, size_t ws_bytes, void *stream) {
    if (M > 0 && (!up || !aligned16(up))) {
        // validate the rest first so that shape errors keep their own status
        const bitnet_status_t st = validate_act(gate, xdt, M, K, gain, fwht, mode, nullptr, nullptr, false);
        return st != BITNET_OK ? st : BITNET_ERR_INVALID_ARG;
    }
    return forward_ws(gate, up, xdt, M, K, gain, eps, fwht, mode, packed, alpha, N, out, false, ws, ws_bytes, stream);
}

size_t bitnet_tl2_bytes(int64_t N, int64_t K) {
    if (N < 0 || K <= 0) return 0;
    return (size_t)N * tl2_row_bytes(K);
}

bitnet_status_t bitnet_pack_tl2(const uint8_t *packed, int64_t N, int64_t K, uint8_t *tl2, void *stream) {
    if (N < 1 || N > kMaxRows) return BITNET_ERR_INVALID_ARG;
    bitnet_status_t st = check_k(K, 0);
    if (st != BITNET_OK) return st;
    if (!packed || !tl2 || !aligned16(packed) || !aligned16(tl2)) return BITNET_ERR_INVALID_ARG;
    return from_cuda(launch_tl2_pack(packed, N, (int)K, tl2, static_cast<cudaStream_t>(stream)));
}

bitnet_status_t bitnet_ternary_gemm_tl2(const int8_t *codes, const float *scale_x, bitnet_act_mode_t mode,
                                        const uint8_t *tl2, const float *alpha, int64_t M, int64_t N, int64_t K,
                                        float *out, int32_t *acc_out, void *stream) {
    bitnet_status_t st = validate_gemm(codes, scale_x, mode, tl2, alpha, M, N, K, out, acc_out);
    if (st != BITNET_OK || M == 0) return st;
    if (M > kGemvMaxM) return BITNET_ERR_UNSUPPORTED_SHAPE;  // a decode format
    return from_cuda(launch_gemv_tl2(codes, scale_x, mode, tl2, alpha, (int)M, (int)N, (int)K, out, acc_out, true,
                                     static_cast<cudaStream_t>(stream)));
}

bitnet_status_t bitnet_hbitlinear_forward_tl2(const void *X, bitnet_dtype_t xdt, int64_t M, int64_t K,
                                              const float *gain, float eps, int fwht, bitnet_act_mode_t mode,
                                              const uint8_t *tl2, const float *alpha, int64_t N, float *out,
                                              void *ws, size_t ws_bytes, void *stream) {
    bitnet_status_t st = validate_forward(X, xdt, M, K, gain, fwht, mode, tl2, alpha, N, out);
    if (st != BITNET_OK || M == 0) return st;
    if (M > kGemvMaxM) return BITNET_ERR_UNSUPPORTED_SHAPE;
    if (!ws || ws_bytes < bitnet_forward_workspace_bytes(M, K) || (reinterpret_cast<uintptr_t>(ws) & 255u))
        return BITNET_ERR_WORKSPACE;
    int8_t *codes = static_cast<int8_t *>(ws);
    float *scale_x = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + align256((size_t)M * (size_t)K));
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = launch_act_quant(X, xdt == BITNET_BF16, M, (int)K, gain, eps, fwht, mode, codes, scale_x, s);
    if (e == cudaSuccess)
        e = launch_gemv_tl2(codes, scale_x, mode, tl2, alpha, (int)M, (int)N, (int)K, out, nullptr, true, s);
    return from_cuda(e);
}

int bitnet_gemm_token_tile(int64_t M, int64_t N, int64_t K) {
    if (M < 0 || N < 1 || N > kMaxRows || check_k(K, 0) != BITNET_OK) return -1;
    if (M <= kGemvMaxM) return 0;
    return gemm_pick_tile((int)M, (int)N, (int)K, sm_count());
}

int bitnet_forward_kernel_count(int64_t M, int64_t N, int64_t K, int fwht, int has_gain) {
    (void)has_gain;
    if (M < 0 || N < 1 || N > kMaxRows || M > kMaxRows || (fwht != 0 && fwht != 1)) return -1;
    if (check_k(K, fwht) != BITNET_OK) return -1;
    return M == 0 ? 0 : 2;  // act_quant, then the decode kernel or the tcgen05 GEMM
}

int bitnet_forward_gemm_plan(int64_t M, int64_t N, int64_t K, int *k_splits) {
    if (k_splits) *k_splits = 0;
    if (M < 0 || N < 1 || N > kMaxRows || check_k(K, 0) != BITNET_OK) return -1;
    if (M <= kGemvMaxM) return 0;
    const GemmPlan p = gemm_plan((int)M, (int)N, (int)K, sm_count(), kSplitCounters);
    if (k_splits) *k_splits = p.splits;
    return p.token_tile;
}

bitnet_status_t bitnet_gemm_force_token_tile(int token_tile) {
    return gemm_force_tile(token_tile) ? BITNET_OK : BITNET_ERR_INVALID_ARG;
}

bitnet_status_t bitnet_gemm_force_k_splits(int k_splits) {
    return gemm_force_splits(k_splits) ? BITNET_OK : BITNET_ERR_INVALID_ARG;
}

bitnet_status_t bitnet_kv_quant(const void *kv, bitnet_dtype_t xdt, int64_t BH, int64_t S, int64_t D, int bits,
                                float eps, int8_t *codes, float *step, float *deq, void *stream) {
    if (xdt != BITNET_F32 && xdt != BITNET_BF16) return BITNET_ERR_INVALID_ARG;
    if (bits != 3 && bits != 4 && bits != 8) return BITNET_ERR_INVALID_ARG;
    if (BH < 0 || S < 0 || BH > kMaxRows || S > kMaxRows || (S > 0 && BH > kMaxRows / S))
        return BITNET_ERR_INVALID_ARG;
    if (D < 4 || D > 1024 || D % 4 != 0) return BITNET_ERR_UNSUPPORTED_SHAPE;
    if (BH == 0 || S == 0) return BITNET_OK;
    if (!kv || !codes || !step || !aligned16(kv) || !aligned16(codes) || !aligned16(step) ||
        (deq && !aligned16(deq)))
        return BITNET_ERR_INVALID_ARG;
    return from_cuda(launch_kv_quant(kv, xdt == BITNET_BF16, BH, S, (int)D, bits, eps, codes, step, deq,
                                     static_cast<cudaStream_t>(stream)));
}

bitnet_status_t bitnet_get_last_device_status(void *stream) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return BITNET_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return BITNET_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return BITNET_ERR_CUDA;
    return static_cast<bitnet_status_t>(v);
}

bitnet_status_t bitnet_selftest_wait_timeout(uint32_t limit_us, void *stream) {
    if (limit_us < 1 || limit_us > 1000000) return BITNET_ERR_INVALID_ARG;
    return from_cuda(launch_wait_selftest(limit_us, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
