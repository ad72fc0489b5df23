/*
 * bitnet.h -- C ABI of libbitnet.so, the B200 (sm_100a) H-BitLinear forward path.
 *
 * The path (BitNet v2 "H-BitLinear", bitnet_v2_engine.py page, Eq. 1-7):
 *   1. per-token RMSNorm,
 *   2. optional Fast Walsh-Hadamard transform along the hidden dimension
 *      (Eq. 3/4, H_m = (1/sqrt2)[[H,H],[H,-H]], natural order),
 *   3. per-token activation quantisation, int8 absmax (Eq. 5) or int4 absmean (Eq. 6),
 *   4. an integer GEMM of those codes against absmean-ternarised weights
 *      (Eq. 1/2) stored at 2 bits per weight,
 *   5. an fp32 dequant epilogue, out = acc * alpha * scale_x / Q.
 *
 * Conventions for every entry point
 *   - Shapes: activations X [M][K], weights W [N][K] (the [out][in] layout of
 *     F.linear), output [M][N]; all row-major and densely packed.
 *   - Pointers: unless stated otherwise every pointer is a DEVICE pointer owned by
 *     the caller.  The library never allocates, frees or retains memory at run time.
 *     Its own device memory is static, allocated when the library is loaded on a
 *     device: one 4-byte status word and the fixed scratch array of
 *     BITNET_NOALLOC_SCRATCH_BYTES (4 MiB) used only by
 *     bitnet_hbitlinear_forward_noalloc.  On the host it keeps per-device caches of
 *     kernel attributes and device addresses.
 *   - Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Every call only enqueues work on that stream and returns without
 *     synchronising; results are ready when the stream reaches them.  The kernels
 *     use programmatic dependent launch: they may begin while the previous kernel on
 *     the stream finishes.  Before their dependency wait they read only the packed
 *     weights (the decode kernel's first loads); they may also issue L2 prefetches
 *     of their other inputs, hints that return no data.  Every other input is read
 *     after the wait.  So
 *     `packed` must not be written by the kernel immediately preceding a call on its
 *     stream, unless that kernel is bitnet_pack_ternary's (it fences its stores) or
 *     ends every writing thread with __threadfence(); copies, events, other streams
 *     and anything earlier are unaffected.  A following kernel launched with
 *     programmatic dependent launch must itself wait (cudaGridDependencySynchronize)
 *     before reading a call's outputs; kernels launched without it start after the
 *     call completes, as usual.
 *   - Errors: every call validates its arguments on the host before launching
 *     anything and returns a bitnet_status_t; nothing throws or aborts.  A kernel
 *     that gives up on a bounded wait records BITNET_ERR_TIMEOUT in the device
 *     status word, which bitnet_get_last_device_status() reads.
 *   - Alignment: every device pointer must be 16-byte aligned (256-byte for
 *     workspaces).  K must be a multiple of 128 and at most 32768 (128 k is the step
 *     of every kernel: one 128-byte row of codes and 32 bytes of packed weights per
 *     row); with the FWHT on K must also be a power of two.  M >= 0 and N >= 1;
 *     M == 0 is a no-op.
 *   - eps is the stabiliser of RMSNorm, of the activation scale and of the weight
 *     scale; the benchmarks use 1e-5.
 */
#ifndef BITNET_H
#define BITNET_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define BITNET_ABI_VERSION 8

#if defined(__GNUC__)
#define BITNET_API __attribute__((visibility("default")))
#else
#define BITNET_API
#endif

typedef enum {
    BITNET_OK = 0,
    BITNET_ERR_INVALID_ARG = 1,       /* null or misaligned pointer, bad enum, negative size */
    BITNET_ERR_UNSUPPORTED_SHAPE = 2, /* K not a multiple of 128, K > 32768, or similar */
    BITNET_ERR_NOT_POW2 = 3,          /* FWHT requested with K not a power of two */
    BITNET_ERR_CUDA = 4,              /* a CUDA runtime call or launch failed */
    BITNET_ERR_TIMEOUT = 5,           /* a kernel gave up on a bounded wait */
    BITNET_ERR_WORKSPACE = 6          /* workspace missing or smaller than required */
} bitnet_status_t;

typedef enum {
    BITNET_ACT_INT8_ABSMAX = 0,  /* Eq. 5: gamma = max|x|, Q = 127, codes in [-128, 127] */
    BITNET_ACT_INT4_ABSMEAN = 1  /* Eq. 6: beta = mean|x|, Q = sqrt(7), codes in [-8, 7] */
} bitnet_act_mode_t;

typedef enum {
    BITNET_F32 = 0,
    BITNET_BF16 = 1
} bitnet_dtype_t;

/*
 * Packed ternary weight layout (this library's format).
 *   Codes: t in {-1, 0, +1} is stored as t + 1 in {0, 1, 2} (the map of the
 *   tl2_lookup_simulation listing in the youngju.dev BitNet transcription); the
 *   value 3 is never written and its meaning is unspecified.
 *   packed is [N][K/4] bytes; row n starts at byte n*K/4.  A row is a sequence of
 *   little-endian 32-bit words; word w holds k in [16w, 16w+16): the code of
 *   k = 16w + 8h + i (h in {0,1}, i in [0,8)) occupies bits [4i+2h, 4i+2h+2) of the
 *   word -- byte 4w + i/2, bit 4(i%2) + 2h.  (One shift and a 0x33333333 mask put
 *   eight codes in eight nibbles; one byte permute makes four of them signed int8.)
 */

/* --------------------------------------------------------------------------
 * bitnet_pack_ternary -- step 4a, once per weight matrix (not on the per-token path).
 * Definition: bitnet_v2_engine.py page, Eq. 1/2 and quantize_weight_ternary:
 *   alpha = mean|W| over all N*K entries (summed in double, one rounding to float),
 *   t = RoundClip(W / (alpha + eps), -1, 1) in fp32, rounding half to even.
 *   W       [N][K] fp32, device, read only.
 *   packed  [N][K/4] bytes, device, written (layout above).
 *   alpha   one fp32, device, written: the per-tensor weight scale used by the GEMM.
 *   ws      device scratch of at least bitnet_pack_workspace_bytes() bytes.
 * Deterministic: the same W always gives the same bytes and alpha.
 * ------------------------------------------------------------------------ */
BITNET_API size_t bitnet_pack_workspace_bytes(int64_t N, int64_t K);
/* One workspace size that serves every call on an M x N x K problem: the largest of
 * bitnet_pack_workspace_bytes(N, K), bitnet_forward_workspace_bytes(M, K) and
 * bitnet_gemm_workspace_bytes(M, N, K). */
BITNET_API size_t bitnet_workspace_bytes(int64_t M, int64_t N, int64_t K);
BITNET_API bitnet_status_t bitnet_pack_ternary(const float *W, int64_t N, int64_t K, float eps,
                                    uint8_t *packed, float *alpha,
                                    void *ws, size_t ws_bytes, void *stream);

/* --------------------------------------------------------------------------
 * bitnet_act_quant -- steps 1-3 fused, one HBM pass per token.
 * Definition: bitnet_v2_engine.py page, HBitLinear.forward (RMSNorm -> Hadamard ->
 * quantise), fast_hadamard_transform (Eq. 3/4), quantize_act_int8 (Eq. 5),
 * quantize_act_int4 (Eq. 6):
 *   r = 1/sqrt(mean(x^2) + eps);  y = (x*r)*gain;  if fwht: y = H_K y;
 *   int8: gamma = max|y|, s = 127/(gamma+eps), code = clamp(rne(y*s), -128, 127);
 *   int4: beta = mean|y|, s = sqrt7/(beta+eps), code = clamp(rne(y*s), -8, 7).
 *   X        [M][K], fp32 or bf16 (xdt), device, read only.
 *   gain     [K] fp32 RMSNorm gain, device; NULL means all ones.
 *   fwht     0 = off, 1 = on (K must then be a power of two: BITNET_ERR_NOT_POW2).
 *   codes    [M][K] int8, device, written (int4 codes are stored one per byte).
 *   scale_x  [M] fp32, device, written: gamma (int8) or beta (int4), without eps.
 * The GPU sums and rotates in a different order than a sequential reference;
 * a code may then differ by one where y*s lies within rounding of a half-integer.
 * ------------------------------------------------------------------------ */
BITNET_API bitnet_status_t bitnet_act_quant(const void *X, bitnet_dtype_t xdt, int64_t M, int64_t K,
                                 const float *gain, float eps, int fwht,
                                 bitnet_act_mode_t mode, int8_t *codes, float *scale_x,
                                 void *stream);

/* --------------------------------------------------------------------------
 * bitnet_ternary_gemm -- steps 4b-5: integer GEMM on packed ternary weights plus
 * the fp32 dequant epilogue.
 * Definition: bitnet_v2_engine.py page, HBitLinear.forward (F.linear of the
 * quantised operands); BitLinear_b158.forward in the youngju.dev transcription
 * (integer product, then output * (w_scale * x_scale) / Q):
 *   acc[m][n] = sum_k codes[m][k] * t[n][k]           (exact int32)
 *   out[m][n] = (float)acc[m][n] * ((alpha * scale_x[m]) / Q),  Q = 127 or sqrt7.
 *   codes    [M][K] int8, device, read only.
 *   scale_x  [M] fp32, device, read only.
 *   packed   [N][K/4] bytes (layout above), device, read only.
 *   alpha    one fp32, device, read only.
 *   out      [M][N] fp32, device, written.
 *   acc_out  [M][N] int32, device, written when not NULL (for exactness checks).
 *   ws       NULL, or device scratch of at least bitnet_gemm_workspace_bytes(M, N, K)
 *            bytes (256-byte aligned; BITNET_ERR_WORKSPACE if smaller).  With a
 *            workspace, a problem with few output tiles for the SMs may split K
 *            over several CTAs per tile as bitnet_hbitlinear_forward does
 *            (bitnet_forward_gemm_plan); the call then first zeroes the workspace's
 *            counters (and, for more than two splits, `out`) with memsets on the
 *            stream.  Without one, K is never split.  The result is bit-identical
 *            either way.
 * M <= 16 runs the weight-streaming decode kernel (tensor-core mma.sync, split-K
 * over the warps of a CTA); larger M runs the persistent tcgen05
 * int8 tensor-core GEMM with TMEM accumulators, whose token-tile size is chosen per
 * shape (see bitnet_gemm_token_tile below).
 * ------------------------------------------------------------------------ */
BITNET_API size_t bitnet_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);
BITNET_API bitnet_status_t bitnet_ternary_gemm(const int8_t *codes, const float *scale_x,
                                    bitnet_act_mode_t mode, const uint8_t *packed,
                                    const float *alpha, int64_t M, int64_t N, int64_t K,
                                    float *out, int32_t *acc_out, void *ws, size_t ws_bytes,
                                    void *stream);

/* --------------------------------------------------------------------------
 * bitnet_hbitlinear_forward -- the whole path: bitnet_act_quant into the
 * workspace, then bitnet_ternary_gemm from it (the second kernel is launched with
 * programmatic dependent launch so its weight stream starts while the first runs).
 * Definition: bitnet_v2_engine.py page, HBitLinear.forward, Eq. 7.
 *   Arguments as in the two calls above; ws is device scratch of at least
 *   bitnet_forward_workspace_bytes(M, K) bytes holding the int8 codes [M][K] at
 *   offset 0 and the per-token scales [M] at offset align256(M*K) between the two
 *   kernels, and 4 KB of tile counters for a split-K GEMM (BITNET_ERR_WORKSPACE if
 *   smaller).  Its contents need no initialisation; after the call the codes and
 *   scales there are the ones the forward used.
 * bitnet_forward_kernel_count: the number of kernels the forward launches for an
 *   M x N x K problem with the FWHT on or off and with or without a gain (2: the
 *   activation kernel and the decode kernel or the tcgen05 GEMM; 0 for M == 0; -1 for
 *   sizes the forward rejects).  Host-only, no CUDA call.
 * ------------------------------------------------------------------------ */
BITNET_API size_t bitnet_forward_workspace_bytes(int64_t M, int64_t K);
BITNET_API int bitnet_forward_kernel_count(int64_t M, int64_t N, int64_t K, int fwht, int has_gain);
BITNET_API bitnet_status_t bitnet_hbitlinear_forward(const void *X, bitnet_dtype_t xdt, int64_t M,
                                          int64_t K, const float *gain, float eps, int fwht,
                                          bitnet_act_mode_t mode, const uint8_t *packed,
                                          const float *alpha, int64_t N, float *out,
                                          void *ws, size_t ws_bytes, void *stream);

/* --------------------------------------------------------------------------
 * bf16-output variants.  The pages' epilogue (bitnet_v2_engine.py page, Eq. 5/6
 * dequantisation; BitLinear_b158.forward's rescale) fixes the value, not the
 * storage type; a bf16 output is this library's storage option.  The same
 * computation as bitnet_ternary_gemm and
 * bitnet_hbitlinear_forward, with the output written as
 *   out_dt == BITNET_F32:   out[m][n] fp32, exactly as the calls above;
 *   out_dt == BITNET_BF16:  out[m][n] = the fp32 value above rounded once to bf16,
 *                           to nearest with ties to even (2 bytes per element),
 * which halves the output stream.  out is [M][N] of out_dt, device, 16-byte
 * aligned; any other out_dt is BITNET_ERR_INVALID_ARG.  The bf16 forward never
 * splits K (its output cannot hold the int32 partial sums), so its plan can differ
 * from bitnet_forward_gemm_plan's for few-tile, long-K shapes; the workspace is
 * the same size.
 * ------------------------------------------------------------------------ */
BITNET_API bitnet_status_t bitnet_ternary_gemm_ex(const int8_t *codes, const float *scale_x,
                                                  bitnet_act_mode_t mode, const uint8_t *packed,
                                                  const float *alpha, int64_t M, int64_t N, int64_t K,
                                                  void *out, bitnet_dtype_t out_dt, int32_t *acc_out,
                                                  void *stream);
BITNET_API bitnet_status_t bitnet_hbitlinear_forward_ex(const void *X, bitnet_dtype_t xdt, int64_t M,
                                                        int64_t K, const float *gain, float eps, int fwht,
                                                        bitnet_act_mode_t mode, const uint8_t *packed,
                                                        const float *alpha, int64_t N, void *out,
                                                        bitnet_dtype_t out_dt, void *ws, size_t ws_bytes,
                                                        void *stream);

/* --------------------------------------------------------------------------
 * SwiGLU-fused variants for the down projection of a BitNet v2 FFN.
 * Definition: bitnet_v2_engine.py page, BitNetV2FFN.forward:
 *   inter = F.silu(gate_proj(x)) * up_proj(x);  out = down_proj(inter)
 * with down_proj an H-BitLinear.  Here the activation step reads gate and up and
 * forms, elementwise in fp32 with one IEEE rounding per operation,
 *   inter[m][k] = (gate / (1 + exp(-gate))) * up        (exp: CUDA expf)
 * in registers; inter is then normalised, rotated and quantised exactly as X is
 * in bitnet_act_quant, and never written to memory.
 *   gate, up  [M][K] in dtype xdt, device, read only (16-byte aligned).
 *   Other arguments, results and errors as for bitnet_act_quant and
 *   bitnet_hbitlinear_forward (the workspace is the same size).
 * ------------------------------------------------------------------------ */
BITNET_API bitnet_status_t bitnet_act_quant_swiglu(const void *gate, const void *up, bitnet_dtype_t xdt, int64_t M,
                                                   int64_t K, const float *gain, float eps, int fwht,
                                                   bitnet_act_mode_t mode, int8_t *codes, float *scale_x,
                                                   void *stream);
BITNET_API bitnet_status_t bitnet_hbitlinear_forward_swiglu(const void *gate, const void *up, bitnet_dtype_t xdt,
                                                            int64_t M, int64_t K, const float *gain, float eps,
                                                            int fwht, bitnet_act_mode_t mode, const uint8_t *packed,
                                                            const float *alpha, int64_t N, float *out, void *ws,
                                                            size_t ws_bytes, void *stream);

/* --------------------------------------------------------------------------
 * bitnet_hbitlinear_forward_noalloc -- the same forward as bitnet_hbitlinear_forward,
 * for callers that cannot allocate device memory: a plugin or extension interface
 * that hands a kernel only its input and output buffers, a runtime that owns all
 * device memory in a preplanned arena, or a latency-critical path that must never
 * reach cudaMalloc (which can synchronise the device).  The paper has no
 * counterpart; this is a deployment variant of the entry point above.
 *   Arguments and results are those of bitnet_hbitlinear_forward without ws/ws_bytes.
 *   The codes and scales between the two kernels live in a fixed array of
 *   BITNET_NOALLOC_SCRATCH_BYTES in the library's own device memory; every GPU that
 *   loads the library holds that array until the process exits.  A call needs
 *   bitnet_forward_workspace_bytes(M, K) <= BITNET_NOALLOC_SCRATCH_BYTES (4 MiB:
 *   for example M*K up to about 4.18 million); larger calls return
 *   BITNET_ERR_WORKSPACE without launching anything.
 *   The call allocates nothing (no cudaMalloc, cudaFree or allocating library
 *   routine).  Its first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call before
 *   any stream capture.
 *   All calls on a device share the one array, which keeps the last call's
 *   contents (nothing in it needs clearing: every code and scale read is first
 *   written by the same call).  Calls that overlap on the GPU -- on different
 *   streams without ordering between them -- race on the array; order them.
 * ------------------------------------------------------------------------ */
#define BITNET_NOALLOC_SCRATCH_BYTES ((size_t)4 << 20)
BITNET_API bitnet_status_t bitnet_hbitlinear_forward_noalloc(const void *X, bitnet_dtype_t xdt, int64_t M,
                                                              int64_t K, const float *gain, float eps, int fwht,
                                                              bitnet_act_mode_t mode, const uint8_t *packed,
                                                              const float *alpha, int64_t N, float *out,
                                                              void *stream);

/* --------------------------------------------------------------------------
 * TL2 weight format: 5 bits per 3 weights (1.67 bits per weight), a decode option.
 * Definition: bitnet_cpp_edge.py page, SignedUnsignedWeightPacker (element-wise mirror
 * consolidation: 27 ternary triplets -> 14 base triplets + a sign bit) and
 * TL2KernelEdge.  Triplet j of a row is (t[3j], t[3j+1], t[3j+2]) (weights past K are
 * 0); read as v = 9 t0 + 3 t1 + t2 in [-13, 13], its index is |v| (the page's base
 * triplets, first nonzero element +1, in order of v) and its sign is v < 0.
 * Layout: row n occupies bitnet_tl2_bytes(1, K) = 20 * ceil(K/96) bytes starting at
 *   n * 20 * ceil(K/96); each group of 32 triplets (96 weights) is 20 bytes: four
 *   little-endian 32-bit index words (triplet 8i + j of the group in bits [4j, 4j+4) of
 *   word i) followed by one little-endian 32-bit sign word (triplet j in bit j).
 * bitnet_pack_tl2: converts 2-bit packed weights (layout above, from
 *   bitnet_pack_ternary) into this format exactly; alpha is unchanged.  packed
 *   [N][K/4] read, tl2 [bitnet_tl2_bytes(N, K)] written, both device, 16-byte aligned.
 * bitnet_ternary_gemm_tl2 / bitnet_hbitlinear_forward_tl2: bitnet_ternary_gemm and
 *   bitnet_hbitlinear_forward with the weights in this format; decode sizes only:
 *   M > 16 returns BITNET_ERR_UNSUPPORTED_SHAPE.  Results are identical to the 2-bit
 *   calls on the same weights (same exact int32 sums, same epilogue).  The decode kernel
 *   looks each triplet's three signed bytes up in a 32-entry shared-memory table
 *   (index | sign << 4), so it spends more instructions per weight than the 2-bit
 *   kernel for 5/6 of its bytes.
 * ------------------------------------------------------------------------ */
BITNET_API size_t bitnet_tl2_bytes(int64_t N, int64_t K);
BITNET_API bitnet_status_t bitnet_pack_tl2(const uint8_t *packed, int64_t N, int64_t K, uint8_t *tl2, void *stream);
BITNET_API bitnet_status_t bitnet_ternary_gemm_tl2(const int8_t *codes, const float *scale_x, bitnet_act_mode_t mode,
                                                   const uint8_t *tl2, const float *alpha, int64_t M, int64_t N,
                                                   int64_t K, float *out, int32_t *acc_out, void *stream);
BITNET_API bitnet_status_t bitnet_hbitlinear_forward_tl2(const void *X, bitnet_dtype_t xdt, int64_t M, int64_t K,
                                                         const float *gain, float eps, int fwht,
                                                         bitnet_act_mode_t mode, const uint8_t *tl2,
                                                         const float *alpha, int64_t N, float *out, void *ws,
                                                         size_t ws_bytes, void *stream);

/* --------------------------------------------------------------------------
 * bitnet_kv_quant -- the low-bit KV cache of a BitNet v2 attention layer.
 * Definition: bitnet_v2_engine.py page, BitNetV2Attention._quantize_kv_head with
 * quantize_act_int8 / quantize_act_int4 (Eq. 5/6).  Per row of D values of a
 * post-RoPE key or value tensor [B][H][S][D] (passed as BH = B*H rows of S tokens):
 *   token s = 0 (BOS, kept at 8 bits):  scale = max|x| + eps,  Q = 127, codes in [-128, 127]
 *   tokens s >= 1, bits = 4:            scale = mean|x| + eps, Q = sqrt7, codes in [-8, 7]
 *   tokens s >= 1, bits = 3:            scale = max|x| + eps,  Q = 3,  codes in [-4, 3]
 *   tokens s >= 1, bits = 8:            as token 0
 *   code = RoundClip(rne((Q / scale) * x)),  step = scale / Q,
 * each an fp32 IEEE operation; step * code is the page's fake-quantised value.
 *   kv     [BH][S][D] fp32 or bf16 (xdt), device, read only.
 *   codes  [BH][S][D] int8, device, written (one code per byte).
 *   step   [BH][S] fp32, device, written.
 *   deq    [BH][S][D] fp32 or NULL: step * code.
 * D must be a multiple of 4 and at most 1024 (BITNET_ERR_UNSUPPORTED_SHAPE);
 * bits other than 3, 4, 8 are BITNET_ERR_INVALID_ARG.  The max of the 3- and 8-bit
 * rows is exact; the mean of the 4-bit rows is summed in another order than a
 * sequential loop, so a 4-bit code may differ by one at a rounding near-tie.
 * ------------------------------------------------------------------------ */
BITNET_API bitnet_status_t bitnet_kv_quant(const void *kv, bitnet_dtype_t xdt, int64_t BH, int64_t S, int64_t D,
                                           int bits, float eps, int8_t *codes, float *step, float *deq,
                                           void *stream);

/* --------------------------------------------------------------------------
 * Prefill GEMM tile control (no counterpart on the pages).
 * bitnet_gemm_token_tile: the token-tile size (256, 224, 192, 128 or 64 tokens
 *   per tensor-core tile) that bitnet_ternary_gemm uses for an M x N x K problem
 *   on the current device; 0 when M <= 16 (the decode kernel runs instead); -1 for
 *   sizes the GEMM rejects.  Includes any forced value.
 * bitnet_forward_gemm_plan: the plan of the GEMM inside bitnet_hbitlinear_forward
 *   (and _noalloc) for the same problem: returns the token tile as above and writes
 *   the k-split count to *k_splits (if not NULL).  When the output has few tiles
 *   for the SMs, the forward splits K over 2, 4 or 8 CTAs per tile.  Two halves:
 *   the first to finish parks its int32 sums in the tile's own output rows and
 *   raises a flag; the second (a CTA of the same grid, already running) waits for
 *   the flag with a bounded wait, adds them and writes the result.  More splits:
 *   the partial int32 sums are added with integer atomics (exact, order-
 *   independent) into `out`, which act_quant zeroes first, and the last split of
 *   each tile dequantises in place.  Either way the result is bit-identical to the
 *   unsplit GEMM on the same codes.
 * bitnet_gemm_force_token_tile: process-wide override of that choice, for every
 *   device and thread: 0 restores the automatic choice; 256, 224, 192, 128 or 64
 *   forces it; any other value returns BITNET_ERR_INVALID_ARG and changes nothing.
 *   Results do not depend on the tile (the int32 accumulators are exact and the
 *   epilogue is elementwise), only the speed does.  For tests and tuning; set it
 *   while no other thread is launching GEMMs.
 * bitnet_gemm_force_k_splits: the same kind of override for the forward's k-split
 *   count: 0 restores the automatic choice; 1, 2, 4 or 8 forces it wherever the
 *   shape allows that count (K/128 divisible by it, at least 4 k-blocks per split,
 *   few enough tiles for the workspace counters); elsewhere the automatic choice
 *   stands.  Any other value returns BITNET_ERR_INVALID_ARG.
 * ------------------------------------------------------------------------ */
BITNET_API int bitnet_gemm_token_tile(int64_t M, int64_t N, int64_t K);
BITNET_API int bitnet_forward_gemm_plan(int64_t M, int64_t N, int64_t K, int *k_splits);
BITNET_API bitnet_status_t bitnet_gemm_force_token_tile(int token_tile);
BITNET_API bitnet_status_t bitnet_gemm_force_k_splits(int k_splits);

/* --------------------------------------------------------------------------
 * Status and diagnostics (no counterpart on the pages).
 * bitnet_status_string: static English text for a status code.
 * bitnet_get_last_device_status: synchronises `stream`, returns the status word
 *   the kernels record on a bounded-wait timeout (BITNET_OK if none) and clears it.
 * bitnet_selftest_wait_timeout: launches one CTA that waits on a barrier nothing
 *   will ever complete, with the given limit in microseconds (1..1000000); the
 *   wait gives up, records BITNET_ERR_TIMEOUT and the kernel returns normally.
 *   Used by the tests to exercise the timeout path without hanging the GPU.
 * bitnet_abi_version: BITNET_ABI_VERSION of the loaded library.
 * ------------------------------------------------------------------------ */
BITNET_API const char *bitnet_status_string(bitnet_status_t status);
BITNET_API bitnet_status_t bitnet_get_last_device_status(void *stream);
BITNET_API bitnet_status_t bitnet_selftest_wait_timeout(uint32_t limit_us, void *stream);
BITNET_API int bitnet_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BITNET_H */
