// kv_quant.cu -- the low-bit KV cache of a BitNet v2 attention layer.
//
// Method: bitnet_v2_engine.py page, BitNetV2Attention._quantize_kv_head with the
// quantisers of Eq. 5/6 (ActQuantINT8STE, ActQuantINT4STE).  Per row of D values
// of a post-RoPE [B, H, S, D] key or value tensor (rows ordered (b, h, s)):
//   token s = 0 (BOS) int8 absmax:  scale = max|x| + eps, code = RoundClip(127 x / scale, -128, 127)
//   tokens s >= 1, bits = 4:        scale = mean|x| + eps, code = RoundClip(sqrt7 x / scale, -8, 7)
//   tokens s >= 1, bits = 3:        scale = max|x| + eps,  code = RoundClip(3 x / scale, -4, 3)
//   tokens s >= 1, bits = 8:        as token 0
// and the dequant step scale / Q, so that step * code is the page's fake-quantised value.
//
// HBM-bound: each input is read once (16-byte loads, several rows in flight per warp),
// the row statistic is a shuffle reduction over the lanes that share the row, and the
// kernel writes D int8 codes, one fp32 step and, when asked, the D dequantised values
// per row.
#include "common.cuh"
#include "host.h"

namespace bitnet {

namespace {

constexpr int KV_WARPS = 8;  // warps per CTA

template <bool BF16>
__device__ __forceinline__ void load4_kv(const void *X, int64_t idx, float *v) {
    if constexpr (BF16) {
        const uint2 u = __ldg(reinterpret_cast<const uint2 *>(reinterpret_cast<const uint16_t *>(X) + idx));
        v[0] = __uint_as_float(u.x << 16);
        v[1] = __uint_as_float(u.x & 0xFFFF0000u);
        v[2] = __uint_as_float(u.y << 16);
        v[3] = __uint_as_float(u.y & 0xFFFF0000u);
    } else {
        const float4 a = __ldg(reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(X) + idx));
        v[0] = a.x;
        v[1] = a.y;
        v[2] = a.z;
        v[3] = a.w;
    }
}

// The code of a clipped product: adding 1.5 * 2^23 rounds to nearest even and leaves
// the integer, two's complement, in the low mantissa bits (|c| < 2^22).
constexpr float kRoundMagic = 12582912.0f;

// Layout: LPR lanes share a row (RP = 32 / LPR rows per warp at a time); lane p of a
// row holds its 4-element groups g = p + LPR * i (i < NG), so each load instruction
// reads LPR * 16 contiguous bytes of every row it touches.  A warp takes IT such row
// sets and issues all their loads before the first reduction, to keep enough bytes in
// flight.  The per-row work (the statistic's last steps, the three divisions, the BOS
// test) is shared by the RP rows of one instruction.
template <bool BF16, int LPR, int NG, int IT>
__global__ void __launch_bounds__(32 * KV_WARPS)
kv_quant_kernel(const void *__restrict__ kv, int64_t rows, int S, int D, int bits, float eps,
                int8_t *__restrict__ codes, float *__restrict__ step, float *__restrict__ deq) {
    constexpr int RP = 32 / LPR;
    pdl_launch_dependents();
    pdl_wait_prerequisites();  // the keys and values come from the previous kernel
    const int lane = threadIdx.x & 31;
    const int p = lane % LPR;
    const int64_t wrow = ((int64_t)blockIdx.x * KV_WARPS + (threadIdx.x >> 5)) * (RP * IT);
    if (wrow >= rows) return;
    const int G = D >> 2;  // 4-element groups in a row
    float v[IT][NG][4];
#pragma unroll
    for (int it = 0; it < IT; ++it) {
        const int64_t r = wrow + it * RP + lane / LPR;
#pragma unroll
        for (int i = 0; i < NG; ++i) {
            const int g = p + LPR * i;
            if (r < rows && g < G) load4_kv<BF16>(kv, r * D + 4 * g, v[it][i]);
            else v[it][i][0] = v[it][i][1] = v[it][i][2] = v[it][i][3] = 0.0f;
        }
    }
    const bool small = rows <= (int64_t)UINT32_MAX;
#pragma unroll
    for (int it = 0; it < IT; ++it) {
        if (wrow + it * RP >= rows) break;  // uniform across the warp
        const int64_t r = wrow + it * RP + lane / LPR;
        const bool live = r < rows;
        const bool bos = small ? ((uint32_t)r % (uint32_t)S == 0u) : (r % S == 0);
        const int rbits = bos ? 8 : bits;
        // rows of one warp instruction may differ in kind (a BOS row beside absmean
        // rows), so every lane takes the same shuffles: the sum or the max is chosen
        // per lane, and xor partners always share the row
        const bool mean = rbits == 4;
        float a = 0.0f;
        if (mean) {
#pragma unroll
            for (int i = 0; i < NG; ++i)
#pragma unroll
                for (int e = 0; e < 4; ++e) a = __fadd_rn(a, fabsf(v[it][i][e]));
        } else {
#pragma unroll
            for (int i = 0; i < NG; ++i)
#pragma unroll
                for (int e = 0; e < 4; ++e) a = fmaxf(a, fabsf(v[it][i][e]));
        }
#pragma unroll
        for (int o = LPR / 2; o > 0; o >>= 1) {
            const float b = __shfl_xor_sync(0xffffffffu, a, o);
            a = mean ? __fadd_rn(a, b) : fmaxf(a, b);
        }
        const float stat = mean ? __fdiv_rn(a, (float)D) : a;
        const float Q = rbits == 8 ? 127.0f : (rbits == 4 ? 2.64575131106459059f : 3.0f);
        const float lo = rbits == 8 ? -128.0f : (rbits == 4 ? -8.0f : -4.0f);
        const float hi = rbits == 8 ? 127.0f : (rbits == 4 ? 7.0f : 3.0f);
        const float scale = __fadd_rn(stat, eps);
        const float sc = __fdiv_rn(Q, scale);
        const float st = __fdiv_rn(scale, Q);
        if (!live) continue;
        if (p == 0) step[r] = st;
#pragma unroll
        for (int i = 0; i < NG; ++i) {
            const int g = p + LPR * i;
            if (g < G) {
                float t[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    t[e] = __fadd_rn(fminf(fmaxf(__fmul_rn(sc, v[it][i][e]), lo), hi), kRoundMagic);
                const uint32_t w01 = __byte_perm(__float_as_uint(t[0]), __float_as_uint(t[1]), 0x0040);
                const uint32_t w23 = __byte_perm(__float_as_uint(t[2]), __float_as_uint(t[3]), 0x0040);
                *reinterpret_cast<uint32_t *>(codes + r * D + 4 * g) = __byte_perm(w01, w23, 0x5410);
                if (deq)  // t - magic is the code as an exact float
                    *reinterpret_cast<float4 *>(deq + r * D + 4 * g) =
                        make_float4(__fmul_rn(st, __fsub_rn(t[0], kRoundMagic)),
                                    __fmul_rn(st, __fsub_rn(t[1], kRoundMagic)),
                                    __fmul_rn(st, __fsub_rn(t[2], kRoundMagic)),
                                    __fmul_rn(st, __fsub_rn(t[3], kRoundMagic)));
            }
        }
    }
}

template <bool BF16, int LPR, int NG, int IT>
cudaError_t launch_kv_cfg(const void *kv, int64_t rows, int S, int D, int bits, float eps, int8_t *codes,
                          float *step, float *deq, cudaStream_t s) {
    constexpr int64_t rows_per_cta = (int64_t)KV_WARPS * (32 / LPR) * IT;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((rows + rows_per_cta - 1) / rows_per_cta));
    cfg.blockDim = dim3(32 * KV_WARPS);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kv_quant_kernel<BF16, LPR, NG, IT>, kv, rows, S, D, bits, eps, codes, step,
                              deq);
}

template <bool BF16>
cudaError_t dispatch_kv(const void *kv, int64_t rows, int S, int D, int bits, float eps, int8_t *codes, float *step,
                        float *deq, cudaStream_t s) {
    // 32 input values per lane in flight (NG * IT = 8 groups of 4)
    if (D <= 32) return launch_kv_cfg<BF16, 8, 1, 8>(kv, rows, S, D, bits, eps, codes, step, deq, s);
    if (D <= 64) return launch_kv_cfg<BF16, 8, 2, 4>(kv, rows, S, D, bits, eps, codes, step, deq, s);
    if (D <= 128) return launch_kv_cfg<BF16, 8, 4, 2>(kv, rows, S, D, bits, eps, codes, step, deq, s);
    if (D <= 256) return launch_kv_cfg<BF16, 16, 4, 2>(kv, rows, S, D, bits, eps, codes, step, deq, s);
    if (D <= 512) return launch_kv_cfg<BF16, 32, 4, 2>(kv, rows, S, D, bits, eps, codes, step, deq, s);
    return launch_kv_cfg<BF16, 32, 8, 1>(kv, rows, S, D, bits, eps, codes, step, deq, s);
}

}  // namespace

cudaError_t launch_kv_quant(const void *kv, bool bf16, int64_t BH, int64_t S, int D, int bits, float eps,
                            int8_t *codes, float *step, float *deq, cudaStream_t s) {
    const int64_t rows = BH * S;
    if (rows == 0) return cudaSuccess;
    return bf16 ? dispatch_kv<true>(kv, rows, (int)S, D, bits, eps, codes, step, deq, s)
                : dispatch_kv<false>(kv, rows, (int)S, D, bits, eps, codes, step, deq, s);
}

}  // namespace bitnet
