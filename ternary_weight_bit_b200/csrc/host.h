// host.h -- host-side declarations shared by the libbitnet translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/bitnet.h"

namespace bitnet {

// Forwards and GEMMs with at most this many tokens run the decode kernel (gemv.cu);
// larger ones the tcgen05 GEMM (gemm_sm100.cu).
constexpr int kGemvMaxM = 16;

// Encode a 2-D tiled TMA descriptor over a row-major byte matrix [rows][row_bytes]
// (element type uint8).  box = {box_x bytes, box_y rows}; swizzle is one of
// CU_TENSOR_MAP_SWIZZLE_{NONE,32B,64B,128B}.  Out-of-bounds boxes read as zero.
bool make_tmap_u8_2d(CUtensorMap *map, const void *base, uint64_t row_bytes, uint64_t rows,
                     uint32_t box_x, uint32_t box_y, CUtensorMapSwizzle swizzle);

// 2D fp32 or bf16 tensor map (no swizzle) over a row-major [rows][cols] array; the row
// pitch and the base must be 16-byte aligned.
bool make_tmap_out_2d(CUtensorMap *map, const void *base, bool bf16, uint64_t cols, uint64_t rows, uint32_t box_x,
                      uint32_t box_y);

// Per-device address of the library's device status word.
int *device_status_ptr();

// Number of SMs of the current device (cached).
int sm_count();

// Optional work for act_quant on behalf of a following split-K GEMM: zero `row_words`
// 32-bit words per token row of `rows` (the GEMM output) and `cnt_n` tile counters.
struct ZeroFill {
    uint32_t *rows = nullptr;
    int row_words = 0;
    int *cnt = nullptr;
    int cnt_n = 0;
};
cudaError_t launch_act_quant(const void *X, bool bf16, int64_t M, int K, const float *gain, float eps,
                             int fwht, int mode, int8_t *codes, float *scale_x, cudaStream_t s,
                             ZeroFill zf = ZeroFill());
// The same with the input formed as the SwiGLU product silu(gate) * up, elementwise.
cudaError_t launch_act_quant_swiglu(const void *gate, const void *up, bool bf16, int64_t M, int K, const float *gain,
                                    float eps, int fwht, int mode, int8_t *codes, float *scale_x, cudaStream_t s,
                                    ZeroFill zf = ZeroFill());

size_t pack_workspace_bytes();
cudaError_t launch_pack(const float *W, int64_t N, int64_t K, float eps, uint8_t *packed, float *alpha,
                        void *ws, cudaStream_t s);

// Decode path (M <= 16): weight-streaming kernel, 2-bit weights unpacked in
// registers, int8 mma.sync, split-K over the warps of one CTA.  `out` is fp32, or
// bf16 when out_bf16 (the fp32 value rounded to nearest even).
cudaError_t launch_gemv(const int8_t *codes, const float *scale_x, int mode, const uint8_t *packed,
                        const float *alpha, int M, int N, int K, void *out, int32_t *acc_out,
                        bool pdl, cudaStream_t s, bool out_bf16 = false);

// TL2 format (1.67 bits per weight): bytes per row, the conversion from the 2-bit
// packed layout (exact) and the decode kernel (M <= 16; out fp32, or bf16 when out_bf16).
size_t tl2_row_bytes(int64_t K);
cudaError_t launch_tl2_pack(const uint8_t *packed, int64_t N, int K, uint8_t *tl2, cudaStream_t s);
cudaError_t launch_gemv_tl2(const int8_t *codes, const float *scale_x, int mode, const uint8_t *tl2,
                            const float *alpha, int M, int N, int K, void *out, int32_t *acc_out, bool pdl,
                            cudaStream_t s, bool out_bf16 = false);

// Prefill path: tcgen05 int8 tensor-core GEMM with TMEM accumulators.
// A plan is a token-tile size (256/224/192/128/64) and a k-split count (1, 2, 4, 8).
// With splits > 2, `out` must be zero on entry (the kernel adds int32 partial sums
// into it before dequantising in place); with splits == 2 it needs no zeroing (the
// pair split below).  With splits > 1, tile_cnt must point at kSplitCounters zeroed
// ints (the kernel leaves them zero again).  A bf16 output
// (out_bf16) is never split.
struct GemmPlan {
    int token_tile;  // 0: choose automatically (no split)
    int splits;
};
constexpr int kSplitCounters = 1024;
// A two-way split ("pair split") keeps per tile an arrival counter (int tile) and a
// ready flag (int kPairFlags + tile) in the same workspace, so it serves up to
// kPairFlags tiles.  The first half to finish parks its int32 sums in the tile's own
// output rows; `out` needs no zeroing then, only the counters.
constexpr int kPairFlags = kSplitCounters / 2;
cudaError_t launch_gemm_tc(const int8_t *codes, const float *scale_x, int mode, const uint8_t *packed,
                           const float *alpha, int M, int N, int K, void *out, int32_t *acc_out,
                           bool pdl, cudaStream_t s, GemmPlan plan = GemmPlan{0, 1}, int *tile_cnt = nullptr,
                           bool out_bf16 = false);

// The plan launch_gemm_tc uses for this shape on `sms` SMs; splits > 1 only when the
// output has at most max_split_tiles tiles (0: never split).  Honors a forced tile.
GemmPlan gemm_plan(int M, int N, int K, int sms, int max_split_tiles);
// Token-tile size of the unsplit plan, and the modelled cost the choice compares.
int gemm_pick_tile(int M, int N, int K, int sms);
double gemm_tile_cost(int bt, int splits, int M, int N, int K, int sms);
// Force the token tile (0 = automatic); false for an unsupported value.
bool gemm_force_tile(int bt);
// Force the forward's k-split count (0 = automatic; 1, 2, 4 or 8) where the shape
// allows it; false for an unsupported value.
bool gemm_force_splits(int splits);

// The forward's kernels (act_quant, then GEMV or GEMM), arguments validated;
// tile_cnt points at kSplitCounters ints of workspace for a split-K GEMM.  With
// `up` given, X is the SwiGLU gate and the input is silu(X) * up.  `out` is fp32,
// or bf16 when out_bf16.
cudaError_t forward_kernels(const void *X, bitnet_dtype_t xdt, int64_t M, int64_t K, const float *gain, float eps,
                            int fwht, bitnet_act_mode_t mode, const uint8_t *packed, const float *alpha,
                            int64_t N, void *out, int8_t *codes, float *scale_x, int *tile_cnt, cudaStream_t s,
                            const void *up = nullptr, bool out_bf16 = false);

// Low-bit KV cache: kv [BH][S][D] (fp32 or bf16), D % 4 == 0, D <= 1024; bits 3, 4 or 8
// for tokens s >= 1 (token 0 is always int8).  deq may be null.
cudaError_t launch_kv_quant(const void *kv, bool bf16, int64_t BH, int64_t S, int D, int bits, float eps,
                            int8_t *codes, float *step, float *deq, cudaStream_t s);

// Argument rules shared by every forward entry point (the workspace is checked by
// each entry point): BITNET_OK or the status the call returns.
bitnet_status_t validate_forward(const void *X, bitnet_dtype_t xdt, int64_t M, int64_t K, const float *gain,
                                 int fwht, bitnet_act_mode_t mode, const uint8_t *packed, const float *alpha,
                                 int64_t N, const void *out);

// Launch the timeout self-test kernel.
cudaError_t launch_wait_selftest(uint32_t limit_us, cudaStream_t s);

}  // namespace bitnet
