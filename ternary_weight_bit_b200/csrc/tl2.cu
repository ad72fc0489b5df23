// tl2.cu -- the TL2 weight format (1.67 bits per weight) and its decode GEMV.
//
// Format: bitnet_cpp_edge.py page, SignedUnsignedWeightPacker and TL2KernelEdge --
// weights are taken three at a time; element-wise mirror consolidation stores each
// triplet as a 4-bit index into the 14 base triplets (first nonzero element +1, and
// the zero triplet) plus one sign bit.  Read as a balanced-ternary number
// v = 9 t0 + 3 t1 + t2, a triplet's index is |v| and its sign is v < 0.  Byte layout
// (include/bitnet.h): per row, groups of 32 triplets (96 weights) of 20 bytes -- four
// 32-bit index words (triplet 8i + j in bits [4j, 4j+4) of word i) and one 32-bit
// sign word (triplet j in bit j); rows padded with zero weights to a multiple of 96.
//
// Decode on B200.  The page's CPU kernel looks sums of activation triplets up in a
// 14-entry table.  Here the tensor cores still do the products (as in the 2-bit
// decode kernel), so the table goes the other way: a 32-entry shared-memory table maps
// (index | sign << 4) to the triplet's three signed bytes, one 32-bit entry per bank,
// so a warp's 32 lookups never conflict.  Three byte permutes turn four looked-up
// triplets into three registers of four consecutive weights.  Lane t of a 4-lane
// quad owns index word t (8 triplets = 24 consecutive k) of a group, i.e. three
// mma.sync.m16n8k32 k-steps of 8 k; the activations are read as the same 24 bytes.
// Structure otherwise as the 2-bit decode kernel (gemv.cu): one CTA per 16 weight
// rows, warps take the groups round-robin with loads several groups ahead, partial
// sums added in shared memory, PDL with the first loads issued before the wait.
#include "common.cuh"
#include "host.h"

namespace bitnet {

namespace {

constexpr int ROWS = 16;        // weight rows per CTA
constexpr int GROUP_K = 96;     // weights per group (32 triplets)
constexpr int GROUP_B = 20;     // bytes per group

__device__ __forceinline__ void mma_s8_16832(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Table entry for code e = index | sign << 4: the triplet's signed bytes (t0, t1, t2, 0);
// 0 for the unused indices 14 and 15.  The digits of the index are its balanced-ternary
// digits, least significant last.
__device__ __forceinline__ uint32_t tl2_entry(int e) {
    const int idx = e & 15;
    if (idx > 13) return 0u;
    int w[3];
    int v = idx;
    for (int d = 2; d >= 0; --d) {
        const int r = (v + 1) % 3 - 1;  // the digit in {-1, 0, 1} congruent to v mod 3
        w[d] = r;
        v = (v - r) / 3;
    }
    const int s = (e >> 4) ? -1 : 1;
    return (uint32_t)(uint8_t)(int8_t)(s * w[0]) | ((uint32_t)(uint8_t)(int8_t)(s * w[1]) << 8) |
           ((uint32_t)(uint8_t)(int8_t)(s * w[2]) << 16);
}

// Eight triplets of one lane (index word, 8 sign bits) -> 24 signed weights in 6 registers.
__device__ __forceinline__ void decode8(uint32_t idxw, uint32_t sgn, const uint32_t *lut, uint32_t (&r)[6]) {
    uint32_t t[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) t[j] = lut[((idxw >> (4 * j)) & 15u) | (((sgn >> j) & 1u) << 4)];
    r[0] = __byte_perm(t[0], t[1], 0x4210);
    r[1] = __byte_perm(t[1], t[2], 0x5421);
    r[2] = __byte_perm(t[2], t[3], 0x6542);
    r[3] = __byte_perm(t[4], t[5], 0x4210);
    r[4] = __byte_perm(t[5], t[6], 0x5421);
    r[5] = __byte_perm(t[6], t[7], 0x6542);
}

template <int NT>
struct Tl2Chunk {
    uint32_t i0, s0, i1, s1;  // index word and sign word of rows g and g+8
    uint2 a[NT][3];           // 24 activation bytes of token 8nt + g
};

template <int WK, int NT, int PF>
__global__ void __launch_bounds__(32 * WK)
gemv_tl2_kernel(const uint8_t *__restrict__ tl2, const int8_t *__restrict__ codes, const float *__restrict__ scale_x,
                const float *__restrict__ alpha, int mode, int M, int N, int K, void *__restrict__ out, int out_bf16,
                int32_t *__restrict__ acc_out) {
    constexpr int TOK = 8 * NT;
    __shared__ uint32_t lut[32];
    __shared__ int32_t red[WK][ROWS * TOK];
    __shared__ float fac[TOK];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int n0 = blockIdx.x * ROWS;
    const int G = (K + GROUP_K - 1) / GROUP_K;
    const int64_t rb = (int64_t)G * GROUP_B;
    const bool v0 = n0 + g < N, v1 = n0 + g + 8 < N;
    const uint8_t *row0 = tl2 + (int64_t)(v0 ? n0 + g : 0) * rb;
    const uint8_t *row1 = tl2 + (int64_t)(v1 ? n0 + g + 8 : 0) * rb;
    if (threadIdx.x < 32) lut[threadIdx.x] = tl2_entry((int)threadIdx.x);

    auto load_w = [&](Tl2Chunk<NT> &ch, int c) {
        const bool in = c < G;
        const uint8_t *p0 = row0 + (int64_t)(in ? c : 0) * GROUP_B, *p1 = row1 + (int64_t)(in ? c : 0) * GROUP_B;
        ch.i0 = (in && v0) ? __ldg(reinterpret_cast<const uint32_t *>(p0) + t) : 0u;
        ch.s0 = (in && v0) ? (__ldg(reinterpret_cast<const uint32_t *>(p0) + 4) >> (8 * t)) & 0xFFu : 0u;
        ch.i1 = (in && v1) ? __ldg(reinterpret_cast<const uint32_t *>(p1) + t) : 0u;
        ch.s1 = (in && v1) ? (__ldg(reinterpret_cast<const uint32_t *>(p1) + 4) >> (8 * t)) & 0xFFu : 0u;
    };
    auto load_act = [&](Tl2Chunk<NT> &ch, int c) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int tok = 8 * nt + g;
            const int64_t kk = (int64_t)GROUP_K * c + 24 * t;
#pragma unroll
            for (int q = 0; q < 3; ++q) {
                const bool in = c < G && tok < M && kk + 8 * q < K;
                ch.a[nt][q] = in ? __ldg(reinterpret_cast<const uint2 *>(codes + (int64_t)tok * K + kk + 8 * q))
                                 : make_uint2(0u, 0u);
            }
        }
    };

    // The packed weights do not depend on the previous kernel (stream contract in
    // bitnet.h): load the first PF groups of every warp before the dependency wait.
    Tl2Chunk<NT> buf[PF];
#pragma unroll
    for (int j = 0; j < PF; ++j) load_w(buf[j], warp + j * WK);
    pdl_launch_dependents();
    pdl_wait_prerequisites();
    if (threadIdx.x < TOK)
        fac[threadIdx.x] = (int)threadIdx.x < M ? dequant_factor(*alpha, __ldg(scale_x + threadIdx.x), mode) : 0.0f;
#pragma unroll
    for (int j = 0; j < PF; ++j) load_act(buf[j], warp + j * WK);
    __syncthreads();  // the table is written

    int acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[nt][e] = 0;

    for (int c0 = warp; c0 < G; c0 += PF * WK) {
#pragma unroll
        for (int j = 0; j < PF; ++j) {
            const int c = c0 + j * WK;
            if (c < G) {
                uint32_t w0[6], w1[6];
                decode8(buf[j].i0, buf[j].s0, lut, w0);
                decode8(buf[j].i1, buf[j].s1, lut, w1);
#pragma unroll
                for (int s = 0; s < 3; ++s)  // k-step: weights 8s..8s+7 of this lane's 24
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                        mma_s8_16832(acc[nt], w0[2 * s], w1[2 * s], w0[2 * s + 1], w1[2 * s + 1], buf[j].a[nt][s].x,
                                     buf[j].a[nt][s].y);
            }
            const int cn = c + PF * WK;  // refill this slot with the group PF rounds ahead
            load_w(buf[j], cn);
            load_act(buf[j], cn);
        }
    }
    // partial sums of this warp: rows g / g+8, tokens 8nt + 2t (+1)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int tk = 8 * nt + 2 * t;
        red[warp][g * TOK + tk] = acc[nt][0];
        red[warp][g * TOK + tk + 1] = acc[nt][1];
        red[warp][(g + 8) * TOK + tk] = acc[nt][2];
        red[warp][(g + 8) * TOK + tk + 1] = acc[nt][3];
    }
    __syncthreads();
    for (int o = threadIdx.x; o < ROWS * TOK; o += 32 * WK) {
        const int tok = o / ROWS, r = o % ROWS;  // consecutive threads -> consecutive n
        const int n = n0 + r;
        if (tok < M && n < N) {
            int32_t sum = 0;
#pragma unroll
            for (int w = 0; w < WK; ++w) sum += red[w][r * TOK + tok];
            const float y = __fmul_rn((float)sum, fac[tok]);
            if (out_bf16)
                reinterpret_cast<__nv_bfloat16 *>(out)[(int64_t)tok * N + n] = __float2bfloat16_rn(y);
            else
                reinterpret_cast<float *>(out)[(int64_t)tok * N + n] = y;
            if (acc_out) acc_out[(int64_t)tok * N + n] = sum;
        }
    }
}

// One thread per (row, group): the 96 weights' 2-bit codes (layout of bitnet.h) to 32
// (index, sign) pairs.  Weights past K are zero.
__global__ void tl2_pack_kernel(const uint8_t *__restrict__ packed, int64_t N, int K, uint8_t *__restrict__ tl2) {
    const int G = (K + GROUP_K - 1) / GROUP_K;
    const int64_t id = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (id >= N * G) return;
    const int64_t n = id / G;
    const int c = (int)(id % G);
    const uint8_t *row = packed + n * (K / 4);
    uint32_t words[5] = {0u, 0u, 0u, 0u, 0u};
    for (int j = 0; j < 32; ++j) {
        int w[3];
        for (int e = 0; e < 3; ++e) {
            const int k = GROUP_K * c + 3 * j + e;
            if (k < K) {
                const uint32_t word = *reinterpret_cast<const uint32_t *>(row + 4 * (k / 16));
                const int h = (k % 16) / 8, i = k % 8;
                w[e] = (int)((word >> (4 * i + 2 * h)) & 3u) - 1;
            } else {
                w[e] = 0;
            }
        }
        const int v = 9 * w[0] + 3 * w[1] + w[2];
        words[j / 8] |= (uint32_t)(v < 0 ? -v : v) << (4 * (j % 8));
        words[4] |= (v < 0 ? 1u : 0u) << j;
    }
    uint32_t *dst = reinterpret_cast<uint32_t *>(tl2 + n * (int64_t)G * GROUP_B + (int64_t)c * GROUP_B);
    for (int i = 0; i < 5; ++i) dst[i] = words[i];
    __threadfence();  // a following decode kernel may read the bytes before its dependency wait
}

template <int WK, int NT, int PF>
cudaError_t launch_tl2_cfg(const uint8_t *tl2, const int8_t *codes, const float *scale_x, int mode,
                           const float *alpha, int M, int N, int K, void *out, bool out_bf16, int32_t *acc_out,
                           bool pdl, cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((N + ROWS - 1) / ROWS));
    cfg.blockDim = dim3(32 * WK);
    cfg.stream = s;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, gemv_tl2_kernel<WK, NT, PF>, tl2, codes, scale_x, alpha, mode, M, N, K, out,
                              out_bf16 ? 1 : 0, acc_out);
}

}  // namespace

size_t tl2_row_bytes(int64_t K) { return K <= 0 ? 0 : (size_t)GROUP_B * (size_t)((K + GROUP_K - 1) / GROUP_K); }

cudaError_t launch_tl2_pack(const uint8_t *packed, int64_t N, int K, uint8_t *tl2, cudaStream_t s) {
    const int G = (K + GROUP_K - 1) / GROUP_K;
    const int64_t total = N * G;
    if (total == 0) return cudaSuccess;
    const int threads = 256;
    tl2_pack_kernel<<<(unsigned)((total + threads - 1) / threads), threads, 0, s>>>(packed, N, K, tl2);
    return cudaGetLastError();
}

cudaError_t launch_gemv_tl2(const int8_t *codes, const float *scale_x, int mode, const uint8_t *tl2,
                            const float *alpha, int M, int N, int K, void *out, int32_t *acc_out, bool pdl,
                            cudaStream_t s, bool out_bf16) {
    const int G = (K + GROUP_K - 1) / GROUP_K;
    const bool wide = G > 32;  // 8 warps per 16 rows when each of 4 would own many groups
    if (M <= 8)
        return wide ? launch_tl2_cfg<8, 1, 3>(tl2, codes, scale_x, mode, alpha, M, N, K, out, out_bf16, acc_out, pdl, s)
                    : launch_tl2_cfg<4, 1, 4>(tl2, codes, scale_x, mode, alpha, M, N, K, out, out_bf16, acc_out, pdl, s);
    return wide ? launch_tl2_cfg<8, 2, 2>(tl2, codes, scale_x, mode, alpha, M, N, K, out, out_bf16, acc_out, pdl, s)
                : launch_tl2_cfg<4, 2, 3>(tl2, codes, scale_x, mode, alpha, M, N, K, out, out_bf16, acc_out, pdl, s);
}

}  // namespace bitnet
