// gemv.cu -- decode path (M <= 16 tokens) of steps 4b-5: stream the 2-bit packed
// ternary weights once from HBM, unpack them in registers and multiply with the
// int8 activation codes on the tensor cores, then apply the dequant epilogue.
//
// Method: bitnet_v2_engine.py page, HBitLinear.forward (F.linear of the quantised
// operands) and Eq. 5/6 for the activation step; BitLinear_b158.forward in the
// youngju.dev BitNet transcription for "integer product, then rescale".
//
// Design (B200).  One CTA per 16 weight rows; its WK warps split K (256-k chunks,
// round-robin) and add their int32 partial sums in shared memory, so no partial sum
// leaves the CTA.  There is no shared-memory staging of the operands: lane (g, t)
// loads, with one 128-bit global load per row, bytes [16t, 16t+16) of the 64-byte
// chunk of rows g and g+8 -- 64 consecutive k -- and the 64 activation bytes of the
// same k for token g.  A dot product does not depend on the order of k, so the MMA's
// k positions are mapped onto those 64 k identically for both operands: k-step s
// (8 per chunk) takes packed word s/2, half s%2 (weights: one mask, one shift and two
// byte permutes per row) and activation bytes 8s..8s+7.  Weights go on the 16-row A
// side of mma.sync m16n8k32 s8, tokens on the 8-column B side.  Each warp keeps up to
// PF chunks of loads in flight.  Launched with programmatic dependent launch, a CTA
// loads its first chunks and bulk-prefetches the rest of its 16 weight rows into L2
// before the dependency wait, so the weight stream overlaps the kernels before it;
// every kernel of the path triggers its dependents at its start.
#include "common.cuh"
#include "host.h"

namespace bitnet {

namespace {

constexpr int ROWS = 16;   // weight rows per CTA

__device__ __forceinline__ void mma_s8_16832(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                             uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 ldg_stream(const uint8_t *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

template <int NT>
struct Chunk {
    uint4 w0, w1;      // 16 bytes of rows g and g+8
    uint4 a[NT][4];    // 64 activation bytes of token 8nt + g
};

template <int WK, int NT, int PF>  // PF: chunks of loads in flight per warp
__global__ void __launch_bounds__(32 * WK)
gemv_kernel(const uint8_t *__restrict__ packed, const int8_t *__restrict__ codes, const float *__restrict__ scale_x,
            const float *__restrict__ alpha, int mode, int M, int N, int K, void *__restrict__ out,
            int out_bf16, int32_t *__restrict__ acc_out) {
    constexpr int TOK = 8 * NT;
    __shared__ int32_t red[WK][ROWS * TOK];
    __shared__ float fac[TOK];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int n0 = blockIdx.x * ROWS;
    const int nch = (K + 255) / 256;
    const int64_t rb = K / 4;  // packed bytes per row
    const bool v0 = n0 + g < N, v1 = n0 + g + 8 < N;
    const uint8_t *wrow0 = packed + (int64_t)(v0 ? n0 + g : 0) * rb + 16 * t;
    const uint8_t *wrow1 = packed + (int64_t)(v1 ? n0 + g + 8 : 0) * rb + 16 * t;

    // Weights do not depend on the previous kernel (see the stream contract in
    // bitnet.h): before the dependency wait, load the first PF chunks of every warp
    // into registers and bulk-prefetch the rest of each of the CTA's 16 rows into L2.
    {
        const int64_t pre = (int64_t)PF * WK * 64;  // bytes of each row the first loads cover
        if (pre < rb && threadIdx.x < ROWS && n0 + (int)threadIdx.x < N)
            bulk_prefetch_l2(packed + (int64_t)(n0 + threadIdx.x) * rb + pre, (uint32_t)(rb - pre));
    }
    Chunk<NT> buf[PF];
#pragma unroll
    for (int j = 0; j < PF; ++j) {
        const int c = warp + j * WK;
        const bool in = c < nch && 64 * c + 16 * t < rb;
        buf[j].w0 = (in && v0) ? ldg_stream(wrow0 + 64 * c) : make_uint4(0, 0, 0, 0);
        buf[j].w1 = (in && v1) ? ldg_stream(wrow1 + 64 * c) : make_uint4(0, 0, 0, 0);
    }
    // The next kernel of the stream may launch now (it waits for this grid before
    // reading anything this grid writes); then wait for the codes and scales.
    pdl_launch_dependents();
    pdl_wait_prerequisites();
    if (threadIdx.x < TOK)
        fac[threadIdx.x] = (int)threadIdx.x < M ? dequant_factor(*alpha, __ldg(scale_x + threadIdx.x), mode) : 0.0f;

    auto load_act = [&](Chunk<NT> &ch, int c) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int tok = 8 * nt + g;
            const int64_t kk = 256 * (int64_t)c + 64 * t;
            const bool in = c < nch && tok < M && kk < K;
            const uint8_t *p = reinterpret_cast<const uint8_t *>(codes) + (int64_t)(in ? tok : 0) * K + (in ? kk : 0);
#pragma unroll
            for (int q = 0; q < 4; ++q)
                ch.a[nt][q] = in ? __ldg(reinterpret_cast<const uint4 *>(p) + q) : make_uint4(0, 0, 0, 0);
        }
    };
#pragma unroll
    for (int j = 0; j < PF; ++j) load_act(buf[j], warp + j * WK);

    int acc[NT][4], acc1[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[nt][e] = acc1[nt][e] = 0;

    for (int c0 = warp; c0 < nch; c0 += PF * WK) {
#pragma unroll
        for (int j = 0; j < PF; ++j) {
            const int c = c0 + j * WK;
            if (c < nch) {
                const Chunk<NT> &ch = buf[j];
                const uint32_t w0[4] = {ch.w0.x, ch.w0.y, ch.w0.z, ch.w0.w};
                const uint32_t w1[4] = {ch.w1.x, ch.w1.y, ch.w1.z, ch.w1.w};
#pragma unroll
                for (int s = 0; s < 8; ++s) {  // k-step: word s/2, half s%2 of this lane's 64 k
                    const int q = s >> 1;
                    const uint32_t m0 = ((s & 1) ? (w0[q] >> 2) : w0[q]) & 0x33333333u;
                    const uint32_t m1 = ((s & 1) ? (w1[q] >> 2) : w1[q]) & 0x33333333u;
                    const uint32_t a0 = ternary4(m0), a2 = ternary4(m0 >> 16);
                    const uint32_t a1 = ternary4(m1), a3 = ternary4(m1 >> 16);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        const uint4 av = ch.a[nt][q];
                        const uint32_t b0 = (s & 1) ? av.z : av.x;
                        const uint32_t b1 = (s & 1) ? av.w : av.y;
                        if (s & 1)
                            mma_s8_16832(acc1[nt], a0, a1, a2, a3, b0, b1);
                        else
                            mma_s8_16832(acc[nt], a0, a1, a2, a3, b0, b1);
                    }
                }
            }
            // refill this slot with the chunk PF rounds ahead
            const int cn = c + PF * WK;
            const bool in = cn < nch && 64 * cn + 16 * t < rb;
            buf[j].w0 = (in && v0) ? ldg_stream(wrow0 + 64 * cn) : make_uint4(0, 0, 0, 0);
            buf[j].w1 = (in && v1) ? ldg_stream(wrow1 + 64 * cn) : make_uint4(0, 0, 0, 0);
            load_act(buf[j], cn);
        }
    }
    // partial sums of this warp: rows g / g+8, tokens 8nt + 2t (+1)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int tk = 8 * nt + 2 * t;
        red[warp][g * TOK + tk] = acc[nt][0] + acc1[nt][0];
        red[warp][g * TOK + tk + 1] = acc[nt][1] + acc1[nt][1];
        red[warp][(g + 8) * TOK + tk] = acc[nt][2] + acc1[nt][2];
        red[warp][(g + 8) * TOK + tk + 1] = acc[nt][3] + acc1[nt][3];
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
            if (out_bf16)  // the fp32 value rounded once, to nearest even
                reinterpret_cast<__nv_bfloat16 *>(out)[(int64_t)tok * N + n] = __float2bfloat16_rn(y);
            else
                reinterpret_cast<float *>(out)[(int64_t)tok * N + n] = y;
            if (acc_out) acc_out[(int64_t)tok * N + n] = sum;
        }
    }
}

template <int WK, int NT, int PF>
cudaError_t launch_cfg(const uint8_t *packed, const int8_t *codes, const float *scale_x, int mode, const float *alpha,
                       int M, int N, int K, void *out, bool out_bf16, int32_t *acc_out, bool pdl, cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((N + ROWS - 1) / ROWS));
    cfg.blockDim = dim3(32 * WK);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, gemv_kernel<WK, NT, PF>, packed, codes, scale_x, alpha, mode, M, N, K, out,
                              out_bf16 ? 1 : 0, acc_out);
}

}  // namespace

cudaError_t launch_gemv(const int8_t *codes, const float *scale_x, int mode, const uint8_t *packed,
                        const float *alpha, int M, int N, int K, void *out, int32_t *acc_out, bool pdl,
                        cudaStream_t s, bool out_bf16) {
    const int nch = (K + 255) / 256;
    // 4 warps per 16-row block for short K, 8 when each warp would otherwise own many chunks
    const int wk = nch <= 16 ? 4 : 8;
    if (M <= 8) {
        if (wk == 4) return launch_cfg<4, 1, 3>(packed, codes, scale_x, mode, alpha, M, N, K, out, out_bf16, acc_out, pdl, s);
        return launch_cfg<8, 1, 2>(packed, codes, scale_x, mode, alpha, M, N, K, out, out_bf16, acc_out, pdl, s);
    }
    if (wk == 4) return launch_cfg<4, 2, 2>(packed, codes, scale_x, mode, alpha, M, N, K, out, out_bf16, acc_out, pdl, s);
    return launch_cfg<8, 2, 2>(packed, codes, scale_x, mode, alpha, M, N, K, out, out_bf16, acc_out, pdl, s);
}

}  // namespace bitnet
