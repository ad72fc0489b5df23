// gemm_sm100.cu -- prefill path of steps 4b-5 on the 5th-generation tensor cores:
// tcgen05.mma kind::i8 (int8 x int8 -> int32) with the accumulator in TMEM.
//
// Method: bitnet_v2_engine.py page, HBitLinear.forward (F.linear of the quantised
// activations and ternary weights); BitLinear_b158.forward in the youngju.dev BitNet
// transcription (integer matrix product, then output * (w_scale * x_scale) / Q).
//
// Tile: 128 tokens (MMA M) x 256 weight rows (MMA N) x 128 k per pipeline stage.
// Warp roles (192 threads):
//   warp 0     TMA producer: activation codes (128x128 B, 128B swizzle) and the packed
//              weight tile (256 rows x 32 B, 32B swizzle) for each stage.
//   warp 1     TMEM allocator; lane 0 issues tcgen05.mma (4 per stage, K = 32 each)
//              and tcgen05.commit.
//   warps 2-5  unpack the 2-bit weights to int8 straight into the K-major 128B-swizzled
//              layout the MMA reads (one mask+shift and one byte permute per 4 weights),
//              fence the generic->async proxy, arrive; then run the epilogue:
//              tcgen05.ld of their 32 TMEM lanes, out = acc * (alpha*scale_x/Q).
// All pipeline waits are bounded; a timeout is recorded in the device status word.
#include "common.cuh"
#include "host.h"

namespace bitnet {

namespace {

constexpr int BM = 128;  // tokens per tile
constexpr int BN = 256;  // weight rows per tile
constexpr int BK = 128;  // k per stage (one 128-byte swizzle row)
constexpr int STAGES = 3;
constexpr int THREADS = 192;
constexpr int A_BYTES = BM * BK;           // 16 KB
constexpr int BU_BYTES = BN * BK;          // 32 KB unpacked int8 weights
constexpr int BP_BYTES = BN * BK / 4;      // 8 KB packed weights
constexpr int A_OFF = 0;
constexpr int BU_OFF = STAGES * A_BYTES;
constexpr int BP_OFF = BU_OFF + STAGES * BU_BYTES;
constexpr int BAR_OFF = BP_OFF + STAGES * BP_BYTES;
constexpr int NUM_BARS = 3 * STAGES + 1;
constexpr int TMEM_SLOT_OFF = BAR_OFF + NUM_BARS * 8;
constexpr int SMEM = TMEM_SLOT_OFF + 16 + 1024;  // + alignment slack
constexpr uint32_t TMEM_COLS = BN;               // 128 lanes x 256 int32 columns

// Instruction descriptor: D = s32, A = s8, B = s8, both K-major, N = 256, M = 128.
constexpr uint32_t kIdesc = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                            ((uint32_t)(BM >> 4) << 24);

// Shared-memory matrix descriptor for a K-major operand in the 128-byte swizzle
// layout: rows of 128 bytes, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);        // start address
    d |= (uint64_t)1 << 16;                          // leading byte offset (unused here)
    d |= (uint64_t)(1024 >> 4) << 32;                // stride byte offset: next 8-row group
    d |= (uint64_t)1 << 46;                          // descriptor version (sm100)
    d |= (uint64_t)2 << 61;                          // swizzle: 128B
    return d;
}

__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}

__device__ __forceinline__ void sts128(uint32_t a, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// 16 weights of one packed word -> 16 signed bytes in k order.
__device__ __forceinline__ uint4 unpack16(uint32_t w) {
    const uint32_t s0 = w & 0x33333333u;         // h = 0: k = 0..7 in nibbles 0..7
    const uint32_t s1 = (w >> 2) & 0x33333333u;  // h = 1: k = 8..15
    return make_uint4(ternary4(s0), ternary4(s0 >> 16), ternary4(s1), ternary4(s1 >> 16));
}

__global__ void __launch_bounds__(THREADS, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
               const float *__restrict__ scale_x, const float *__restrict__ alpha, int mode, int M, int N,
               int K, float *__restrict__ out, int32_t *__restrict__ acc_out, int *status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + BAR_OFF);
    uint64_t *unpacked = full + STAGES;
    uint64_t *empty = unpacked + STAGES;
    uint64_t *accfull = empty + STAGES;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + TMEM_SLOT_OFF);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * BN;
    const int m0 = blockIdx.y * BM;
    const int KB = K / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&unpacked[s], 4);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accfull, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_d = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tm_a);
            tma_prefetch_desc(&tm_b);
            const int pre = KB < STAGES ? KB : STAGES;
            for (int kb = 0; kb < pre; ++kb) {
                mbar_arrive_expect_tx(&full[kb], A_BYTES + BP_BYTES);
                tma_load_2d(smem + BP_OFF + kb * BP_BYTES, &tm_b, &full[kb], kb * (BK / 4), n0);
            }
            pdl_wait_prerequisites();  // activation codes come from the previous kernel
            for (int kb = 0; kb < pre; ++kb)
                tma_load_2d(smem + A_OFF + kb * A_BYTES, &tm_a, &full[kb], kb * BK, m0);
            int issued = pre;
            for (int kb = STAGES; kb < KB; ++kb) {
                const int s = kb % STAGES;
                if (!mbar_wait(&empty[s], ((kb / STAGES) - 1) & 1, status)) break;
                mbar_arrive_expect_tx(&full[s], A_BYTES + BP_BYTES);
                tma_load_2d(smem + BP_OFF + s * BP_BYTES, &tm_b, &full[s], kb * (BK / 4), n0);
                tma_load_2d(smem + A_OFF + s * A_BYTES, &tm_a, &full[s], kb * BK, m0);
                issued = kb + 1;
            }
            const int last = issued - 1;  // every issued load must land before exit
            for (int s = 0; s < STAGES && s <= last; ++s) {
                const int li = last - ((last - s) % STAGES);
                mbar_wait(&full[s], (li / STAGES) & 1, status);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            for (int kb = 0; kb < KB; ++kb) {
                const int s = kb % STAGES;
                const uint32_t par = (kb / STAGES) & 1;
                if (!mbar_wait(&full[s], par, status)) break;
                if (!mbar_wait(&unpacked[s], par, status)) break;
                tc_fence_after();
                const uint32_t a_addr = smem_u32(smem + A_OFF + s * A_BYTES);
                const uint32_t b_addr = smem_u32(smem + BU_OFF + s * BU_BYTES);
                const uint64_t adesc = smem_desc_sw128(a_addr);
                const uint64_t bdesc = smem_desc_sw128(b_addr);
#pragma unroll
                for (int j = 0; j < BK / 32; ++j) {
                    // advance 32 bytes of K inside the swizzled 128-byte rows
                    umma_i8(tmem_d, adesc + (uint64_t)(2 * j), bdesc + (uint64_t)(2 * j), kIdesc,
                            (kb | j) != 0 ? 1u : 0u);
                }
                umma_commit(&empty[s]);  // stage s may be refilled once these MMAs finish
            }
            umma_commit(accfull);
        }
    } else {
        // ------------------------------------------------------------ unpack, then epilogue
        const int ut = threadIdx.x - 64;  // 0..127
        for (int kb = 0; kb < KB; ++kb) {
            const int s = kb % STAGES;
            if (kb >= STAGES && !mbar_wait(&empty[s], ((kb / STAGES) - 1) & 1, status)) break;
            if (!mbar_wait(&full[s], (kb / STAGES) & 1, status)) break;
            const uint32_t bp = smem_u32(smem + BP_OFF + s * BP_BYTES);
            const uint32_t bu = smem_u32(smem + BU_OFF + s * BU_BYTES);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int n = ut + 128 * half;  // row of the weight tile
                // packed row: 32 bytes, 32B swizzle (16-byte chunk index ^= bit 2 of the row)
                const int sw = (n >> 2) & 1;
                const uint4 p0 = lds128(bp + n * 32 + ((0 ^ sw) << 4));
                const uint4 p1 = lds128(bp + n * 32 + ((1 ^ sw) << 4));
                const uint32_t w[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
                const uint32_t row = bu + (n >> 3) * 1024 + (n & 7) * 128;
#pragma unroll
                for (int c = 0; c < 8; ++c) sts128(row + ((c ^ (n & 7)) << 4), unpack16(w[c]));
            }
            fence_proxy_async_smem();  // make the generic-proxy writes visible to tcgen05.mma
            __syncwarp();
            if (lane == 0) mbar_arrive(&unpacked[s]);
        }

        // epilogue: this warp may touch TMEM lanes [32*(warp%4), +32)
        const int q = warp & 3;
        const int m = m0 + 32 * q + lane;
        mbar_wait(accfull, 0, status);
        tc_fence_after();
        pdl_wait_prerequisites();
        const float f = m < M ? dequant_factor(*alpha, __ldg(scale_x + m), mode) : 0.0f;
        const uint32_t taddr = tmem_d + ((uint32_t)(32 * q) << 16);
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
            uint32_t r[32];
            tmem_ld_32x32b_x32(taddr + 32 * c, r);
            tmem_wait_ld();
            if (m < M) {
                const int nb = n0 + 32 * c;
                float *orow = out + (int64_t)m * N + nb;
                if (nb + 32 <= N && (N & 3) == 0) {
#pragma unroll
                    for (int j = 0; j < 32; j += 4) {
                        const float4 v = make_float4(__fmul_rn((float)(int)r[j], f), __fmul_rn((float)(int)r[j + 1], f),
                                                     __fmul_rn((float)(int)r[j + 2], f), __fmul_rn((float)(int)r[j + 3], f));
                        *reinterpret_cast<float4 *>(orow + j) = v;
                    }
                    if (acc_out) {
                        int32_t *arow = acc_out + (int64_t)m * N + nb;
#pragma unroll
                        for (int j = 0; j < 32; j += 4)
                            *reinterpret_cast<int4 *>(arow + j) =
                                make_int4((int)r[j], (int)r[j + 1], (int)r[j + 2], (int)r[j + 3]);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        if (nb + j < N) {
                            orow[j] = __fmul_rn((float)(int)r[j], f);
                            if (acc_out) acc_out[(int64_t)m * N + nb + j] = (int)r[j];
                        }
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_d, TMEM_COLS);
    }
}

}  // namespace

cudaError_t launch_gemm_tc(const int8_t *codes, const float *scale_x, int mode, const uint8_t *packed,
                           const float *alpha, int M, int N, int K, float *out, int32_t *acc_out, bool pdl,
                           cudaStream_t s) {
    CUtensorMap ta, tb;
    if (!make_tmap_u8_2d(&ta, codes, (uint64_t)K, (uint64_t)M, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (!make_tmap_u8_2d(&tb, packed, (uint64_t)K / 4, (uint64_t)N, BK / 4, BN, CU_TENSOR_MAP_SWIZZLE_32B))
        return cudaErrorInvalidValue;
    static bool done[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= kMaxDevices || !done[dev]) {
        e = cudaFuncSetAttribute(gemm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
        if (e != cudaSuccess) return e;
        if (dev < kMaxDevices) done[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((N + BN - 1) / BN), (unsigned)((M + BM - 1) / BM));
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = SMEM;
    cfg.stream = s;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, gemm_tc_kernel, ta, tb, scale_x, alpha, mode, M, N, K, out, acc_out,
                              device_status_ptr());
}

}  // namespace bitnet
