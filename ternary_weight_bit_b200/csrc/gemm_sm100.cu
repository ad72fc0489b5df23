// gemm_sm100.cu -- prefill path of steps 4b-5 on the 5th-generation tensor cores:
// tcgen05.mma kind::i8 (int8 x int8 -> int32) with the accumulator in TMEM.
//
// Method: bitnet_v2_engine.py page, HBitLinear.forward (F.linear of the quantised
// activations and ternary weights); BitLinear_b158.forward in the youngju.dev BitNet
// transcription (integer matrix product, then output * (w_scale * x_scale) / Q).
//
// The MMA computes D[n][m] = sum_k t[n][k] * q[m][k] with the weights on its M side:
//   A = 128 ternary weight rows, unpacked from 2 bits straight into TMEM with
//       tcgen05.st (they never pass through shared memory);
//   B = BT activation-code rows (tokens), TMA-loaded into shared memory in the
//       K-major 128-byte-swizzled layout;
//   D = 128 lanes (weight rows) x BT int32 columns (tokens) in TMEM.
// Per 128-k stage the shared memory only carries the activation tile (BT x 128 B)
// and the packed weights (128 x 32 B).
//
// Warp roles (192 threads):
//   warp 0     TMA producer (activation tile, 128B swizzle; packed weights, 32B swizzle)
//   warp 1     TMEM allocator; lane 0 issues 4 x tcgen05.mma per stage and the commits
//   warps 2-5  each owns the 32 TMEM lanes (weight rows) of its lane quarter: unpack
//              its rows into the stage's A columns, then run the epilogue
//              (tcgen05.ld, out[m][n] = acc * f[m], stores coalesced along n).
// All waits are bounded; a timeout is recorded in the device status word.
#include "common.cuh"
#include "host.h"

namespace bitnet {

namespace {

constexpr int BW = 128;  // weight rows per tile (MMA M)
constexpr int BK = 128;  // k per stage
constexpr int THREADS = 192;

template <int BT>
struct TcCfg {
    static constexpr int STAGES = BT >= 256 ? 4 : 6;
    static constexpr int CTAS_PER_SM = BT <= 64 ? 2 : 1;
    static constexpr int B_BYTES = BT * BK;        // activation tile
    static constexpr int P_BYTES = BW * BK / 4;    // packed weight tile (4 KB)
    static constexpr int B_OFF = 0;
    static constexpr int P_OFF = STAGES * B_BYTES;
    static constexpr int F_OFF = P_OFF + STAGES * P_BYTES;  // per-token dequant factors
    static constexpr int BAR_OFF = F_OFF + BT * 4;
    static constexpr int NUM_BARS = 3 * STAGES + 1;
    static constexpr int TMEM_SLOT_OFF = BAR_OFF + NUM_BARS * 8;
    static constexpr int SMEM = TMEM_SLOT_OFF + 16 + 1024;
    // D: BT columns, A stages: 32 columns each; allocations are powers of two.
    static constexpr uint32_t TMEM_COLS = (BT + 32 * STAGES) <= 256 ? 256 : 512;
    static constexpr uint32_t A_COL0 = BT;
    static_assert(BT + 32 * STAGES <= (int)TMEM_COLS, "TMEM budget");
    static_assert(CTAS_PER_SM * TMEM_COLS <= 512, "co-resident CTAs must fit in TMEM together");
    // D = s32, A = s8, B = s8, K-major both, N = BT, M = 128.
    static constexpr uint32_t IDESC = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BT >> 3) << 17) |
                                      ((uint32_t)(BW >> 4) << 24);
};

__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);  // start address
    d |= (uint64_t)1 << 16;                    // leading byte offset (unused for swizzled K-major)
    d |= (uint64_t)(1024 >> 4) << 32;          // stride byte offset: next 8-row group
    d |= (uint64_t)1 << 46;                    // descriptor version (sm100)
    d |= (uint64_t)2 << 61;                    // swizzle: 128B
    return d;
}

__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}

// D[tmem] (+)= A[tmem] * B[smem desc]^T, int8 x int8 -> int32.
__device__ __forceinline__ void umma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
        "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
        "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

template <int BT>
__global__ void __launch_bounds__(THREADS, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_act, const __grid_constant__ CUtensorMap tm_w,
               const float *__restrict__ scale_x, const float *__restrict__ alpha, int mode, int M, int N, int K,
               float *__restrict__ out, int32_t *__restrict__ acc_out, int *status) {
    using C = TcCfg<BT>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
    uint64_t *unpacked = full + C::STAGES;
    uint64_t *empty = unpacked + C::STAGES;
    uint64_t *accfull = empty + C::STAGES;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::TMEM_SLOT_OFF);
    float *fac = reinterpret_cast<float *>(smem + C::F_OFF);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * BW;  // weight rows
    const int m0 = blockIdx.y * BT;  // tokens
    const int KB = K / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&unpacked[s], 4);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accfull, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tm_act);
            tma_prefetch_desc(&tm_w);
            const int pre = KB < C::STAGES ? KB : C::STAGES;
            for (int kb = 0; kb < pre; ++kb) {
                mbar_arrive_expect_tx(&full[kb], C::B_BYTES + C::P_BYTES);
                tma_load_2d(smem + C::P_OFF + kb * C::P_BYTES, &tm_w, &full[kb], kb * (BK / 4), n0);
            }
            pdl_wait_prerequisites();  // activation codes come from the previous kernel
            for (int kb = 0; kb < pre; ++kb)
                tma_load_2d(smem + C::B_OFF + kb * C::B_BYTES, &tm_act, &full[kb], kb * BK, m0);
            int issued = pre;
            for (int kb = C::STAGES; kb < KB; ++kb) {
                const int s = kb % C::STAGES;
                if (!mbar_wait(&empty[s], ((kb / C::STAGES) - 1) & 1, status)) break;
                mbar_arrive_expect_tx(&full[s], C::B_BYTES + C::P_BYTES);
                tma_load_2d(smem + C::P_OFF + s * C::P_BYTES, &tm_w, &full[s], kb * (BK / 4), n0);
                tma_load_2d(smem + C::B_OFF + s * C::B_BYTES, &tm_act, &full[s], kb * BK, m0);
                issued = kb + 1;
            }
            const int last = issued - 1;  // every issued load must land before exit
            for (int s = 0; s < C::STAGES && s <= last; ++s) {
                const int li = last - ((last - s) % C::STAGES);
                mbar_wait(&full[s], (li / C::STAGES) & 1, status);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            for (int kb = 0; kb < KB; ++kb) {
                const int s = kb % C::STAGES;
                const uint32_t par = (kb / C::STAGES) & 1;
                if (!mbar_wait(&full[s], par, status)) break;
                if (!mbar_wait(&unpacked[s], par, status)) break;
                tc_fence_after();
                const uint64_t bdesc = smem_desc_sw128(smem_u32(smem + C::B_OFF + s * C::B_BYTES));
                const uint32_t a_tmem = tmem_base + C::A_COL0 + 32 * s;
#pragma unroll
                for (int j = 0; j < BK / 32; ++j)  // K = 32 per MMA: 8 TMEM columns of A, 32 bytes of B rows
                    umma_i8_ts(tmem_base, a_tmem + 8 * j, bdesc + (uint64_t)(2 * j), C::IDESC,
                               (kb | j) != 0 ? 1u : 0u);
                umma_commit(&empty[s]);  // the stage (A columns and B tile) is free once these finish
            }
            umma_commit(accfull);
        }
    } else {
        // ------------------------------------------------------------ unpack into TMEM, then epilogue
        const int q = warp & 3;            // TMEM lane quarter of this warp
        const int r = 32 * q + lane;       // weight row within the tile (= TMEM lane)
        const uint32_t lane_off = (uint32_t)(32 * q) << 16;
        pdl_wait_prerequisites();
        for (int i = threadIdx.x - 64; i < BT; i += 128) {
            const int m = m0 + i;
            fac[i] = m < M ? dequant_factor(*alpha, __ldg(scale_x + m), mode) : 0.0f;
        }
        const int sw = (r >> 2) & 1;  // 32B swizzle of the packed row
        for (int kb = 0; kb < KB; ++kb) {
            const int s = kb % C::STAGES;
            if (kb >= C::STAGES && !mbar_wait(&empty[s], ((kb / C::STAGES) - 1) & 1, status)) break;
            if (!mbar_wait(&full[s], (kb / C::STAGES) & 1, status)) break;
            const uint32_t bp = smem_u32(smem + C::P_OFF + s * C::P_BYTES) + r * 32;
            const uint4 p0 = lds128(bp + ((0 ^ sw) << 4));
            const uint4 p1 = lds128(bp + ((1 ^ sw) << 4));
            const uint32_t w[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
            uint32_t a[32];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint32_t s0 = w[c] & 0x33333333u;         // k = 16c + 0..7
                const uint32_t s1 = (w[c] >> 2) & 0x33333333u;  // k = 16c + 8..15
                a[4 * c + 0] = ternary4(s0);
                a[4 * c + 1] = ternary4(s0 >> 16);
                a[4 * c + 2] = ternary4(s1);
                a[4 * c + 3] = ternary4(s1 >> 16);
            }
            tc_fence_after();  // order after the MMA that freed this stage
            tmem_st_32x32b_x32(tmem_base + lane_off + C::A_COL0 + 32 * s, a);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&unpacked[s]);
        }

        // epilogue: TMEM lane r holds weight row n0 + r, column j token m0 + j
        mbar_wait(accfull, 0, status);
        tc_fence_after();
        asm volatile("bar.sync 1, 128;" ::: "memory");  // the four unpack warps: fac[] is complete
        const int n = n0 + r;
#pragma unroll 1
        for (int c = 0; c < BT / 32; ++c) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(tmem_base + lane_off + 32 * c, v);
            tmem_wait_ld();
            if (n < N) {
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int m = m0 + 32 * c + j;
                    if (m < M) {
                        out[(int64_t)m * N + n] = __fmul_rn((float)(int)v[j], fac[32 * c + j]);
                        if (acc_out) acc_out[(int64_t)m * N + n] = (int)v[j];
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

template <int BT>
cudaError_t launch_bt(const int8_t *codes, const float *scale_x, int mode, const uint8_t *packed, const float *alpha,
                      int M, int N, int K, float *out, int32_t *acc_out, bool pdl, cudaStream_t s) {
    using C = TcCfg<BT>;
    CUtensorMap ta, tw;
    if (!make_tmap_u8_2d(&ta, codes, (uint64_t)K, (uint64_t)M, BK, BT, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (!make_tmap_u8_2d(&tw, packed, (uint64_t)K / 4, (uint64_t)N, BK / 4, BW, CU_TENSOR_MAP_SWIZZLE_32B))
        return cudaErrorInvalidValue;
    auto kern = gemm_tc_kernel<BT>;
    static bool done[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= kMaxDevices || !done[dev]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (e != cudaSuccess) return e;
        if (dev < kMaxDevices) done[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((N + BW - 1) / BW), (unsigned)((M + BT - 1) / BT));
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = s;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, ta, tw, scale_x, alpha, mode, M, N, K, out, acc_out, device_status_ptr());
}

}  // namespace

// Relative cost of a token tile size: waves of CTAs times the per-tile work, over
// the tile's efficiency (smaller tiles move more shared-memory bytes and unpack
// more weights per MAC).
double tile_cost(int BT, int M, int N, int sms) {
    const double eff = BT >= 256 ? 1.0 : (BT >= 128 ? 0.85 : 0.65);
    const int per_sm = BT <= 64 ? 2 : 1;
    const long tiles = (long)((N + BW - 1) / BW) * ((M + BT - 1) / BT);
    const long waves = (tiles + (long)sms * per_sm - 1) / ((long)sms * per_sm);
    return (double)waves * BT / eff;
}

cudaError_t launch_gemm_tc(const int8_t *codes, const float *scale_x, int mode, const uint8_t *packed,
                           const float *alpha, int M, int N, int K, float *out, int32_t *acc_out, bool pdl,
                           cudaStream_t s) {
    const int sms = sm_count();
    int bt = 256;
    double best = tile_cost(256, M, N, sms);
    if (tile_cost(128, M, N, sms) < best) {
        bt = 128;
        best = tile_cost(128, M, N, sms);
    }
    if (M <= 64 && tile_cost(64, M, N, sms) < best) bt = 64;
    if (bt == 256) return launch_bt<256>(codes, scale_x, mode, packed, alpha, M, N, K, out, acc_out, pdl, s);
    if (bt == 128) return launch_bt<128>(codes, scale_x, mode, packed, alpha, M, N, K, out, acc_out, pdl, s);
    return launch_bt<64>(codes, scale_x, mode, packed, alpha, M, N, K, out, acc_out, pdl, s);
}

}  // namespace bitnet
