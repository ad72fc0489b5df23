// gemv.cu -- decode path (M <= 16 tokens) of steps 4b-5: stream the 2-bit packed
// ternary weights once from HBM, unpack them in registers and multiply with the
// int8 activation codes on the tensor cores, then apply the dequant epilogue.
//
// Method: bitnet_v2_engine.py page, HBitLinear.forward (F.linear of the quantised
// operands) and Eq. 5/6 for the activation step; BitLinear_b158.forward in the
// youngju.dev BitNet transcription for "integer product, then rescale".
//
// Design (B200):
//   * Work unit = 16*WARPS weight rows x a K-slice.  The CTAs of one thread-block
//     cluster share a row block and split K; their int32 partial sums are added
//     through distributed shared memory (exact), so no global scratch is used.
//   * One producer lane streams 256-k stages with TMA: the packed weight tile
//     (64-byte rows, 64B swizzle) and the activation codes (two 128-byte boxes,
//     128B swizzle), into a STAGES-deep mbarrier ring.  The weight loads of the
//     first stages are issued before griddepcontrol.wait, so with programmatic
//     dependent launch they overlap the activation-quantisation kernel.
//   * Each compute warp owns 16 weight rows.  mma.sync m16n8k32 s8 is used "swap-AB":
//     weights fill the 16-row A side, tokens the 8-column B side.  A weight
//     fragment is built from the packed word with one shift, one mask and one byte
//     permute per 4 weights.  Accumulation is exact int32.
#include "common.cuh"
#include "host.h"

namespace bitnet {

namespace {

template <int WARPS, int NT>
struct GemvCfg {
    static constexpr int ROWS = 16 * WARPS;  // weight rows per CTA
    static constexpr int TOK = 8 * NT;       // token rows (M padded)
    static constexpr int KSTAGE = 256;       // k per pipeline stage
    static constexpr int W_BYTES = ROWS * 64;
    static constexpr int A_BOX = TOK * 128;  // one 128-k activation box
    static constexpr int A_BYTES = 2 * A_BOX;
    static constexpr int W_OFF = 0;
    static constexpr int A_OFF = (W_BYTES + 1023) / 1024 * 1024;
    static constexpr int STAGE = A_OFF + (A_BYTES + 1023) / 1024 * 1024;
    static constexpr int STAGES = 6;
    static constexpr int THREADS = 32 * (WARPS + 1);
    static constexpr int BAR_OFF = STAGES * STAGE;
    static constexpr int RED_OFF = BAR_OFF + 2 * STAGES * 8;
    static constexpr int SMEM = RED_OFF + ROWS * TOK * 4 + 1024;  // + alignment slack
};

__device__ __forceinline__ uint4 lds128(const uint8_t *p) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(smem_u32(p)));
    return v;
}

__device__ __forceinline__ uint32_t lds32(const uint8_t *p) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)));
    return v;
}

__device__ __forceinline__ void mma_s8_16832(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                             uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}

__device__ __forceinline__ int32_t ld_dsmem_s32(const int32_t *p, uint32_t rank) {
    uint32_t ra;
    int32_t v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(p)), "r"(rank));
    asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(ra) : "memory");
    return v;
}

template <int WARPS, int NT>
__global__ void __launch_bounds__(GemvCfg<WARPS, NT>::THREADS)
gemv_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_a,
            const float *__restrict__ scale_x, const float *__restrict__ alpha, int mode, int M, int N,
            int K, int nsplit, float *__restrict__ out, int32_t *__restrict__ acc_out, int *status) {
    using C = GemvCfg<WARPS, NT>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
    uint64_t *empty = full + C::STAGES;
    int32_t *red = reinterpret_cast<int32_t *>(smem + C::RED_OFF);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t split = nsplit > 1 ? cluster_ctarank() : 0;
    const int n0 = (int)(blockIdx.x / nsplit) * C::ROWS;
    const int nch = (K + C::KSTAGE - 1) / C::KSTAGE;
    const int c0 = (int)((int64_t)split * nch / nsplit);
    const int c1 = (int)((int64_t)(split + 1) * nch / nsplit);
    const int my = c1 - c0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], WARPS);
        }
        fence_mbar_init();
    }
    __syncthreads();

    int acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0;

    if (warp == WARPS) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            tma_prefetch_desc(&tm_w);
            tma_prefetch_desc(&tm_a);
            const int pre = my < C::STAGES ? my : C::STAGES;
            for (int i = 0; i < pre; ++i) {
                uint8_t *st = smem + i * C::STAGE;
                mbar_arrive_expect_tx(&full[i], C::W_BYTES + C::A_BYTES);
                tma_load_2d(st + C::W_OFF, &tm_w, &full[i], (c0 + i) * 64, n0);
            }
            pdl_wait_prerequisites();  // the activation codes come from the previous kernel
            for (int i = 0; i < pre; ++i) {
                uint8_t *st = smem + i * C::STAGE;
                tma_load_2d(st + C::A_OFF, &tm_a, &full[i], (c0 + i) * C::KSTAGE, 0);
                tma_load_2d(st + C::A_OFF + C::A_BOX, &tm_a, &full[i], (c0 + i) * C::KSTAGE + 128, 0);
            }
            bool ok = true;
            int issued = pre;
            for (int i = C::STAGES; i < my && ok; ++i) {
                const int s = i % C::STAGES;
                ok = mbar_wait(&empty[s], ((i / C::STAGES) - 1) & 1, status);
                if (!ok) break;
                uint8_t *st = smem + s * C::STAGE;
                mbar_arrive_expect_tx(&full[s], C::W_BYTES + C::A_BYTES);
                tma_load_2d(st + C::W_OFF, &tm_w, &full[s], (c0 + i) * 64, n0);
                tma_load_2d(st + C::A_OFF, &tm_a, &full[s], (c0 + i) * C::KSTAGE, 0);
                tma_load_2d(st + C::A_OFF + C::A_BOX, &tm_a, &full[s], (c0 + i) * C::KSTAGE + 128, 0);
                issued = i + 1;
            }
            // Before this CTA may exit, every load it issued must have landed.
            const int last = issued - 1;
            for (int s = 0; s < C::STAGES && s <= last; ++s) {
                const int li = last - ((last - s) % C::STAGES);  // last load issued on stage s
                mbar_wait(&full[s], (li / C::STAGES) & 1, status);
            }
        }
    } else {
        // ---------------------------------------------------------- compute warps
        pdl_wait_prerequisites();
        const int g = lane >> 2, t = lane & 3;
        const int sh = 2 * (t >> 1) + 16 * (t & 1);  // selects this lane's 4 codes of a word
        const int r0 = warp * 16 + g, r1 = r0 + 8;
        const int sw0 = (r0 >> 1) & 3, sw1 = (r1 >> 1) & 3;  // 64B swizzle of rows r0, r1
        for (int i = 0; i < my; ++i) {
            const int s = i % C::STAGES;
            if (!mbar_wait(&full[s], (i / C::STAGES) & 1, status)) break;
            const uint8_t *ws = smem + s * C::STAGE + C::W_OFF;
            const uint8_t *as = smem + s * C::STAGE + C::A_OFF;
#pragma unroll
            for (int c = 0; c < 4; ++c) {  // 64-k chunks of the stage
                const uint4 lo = lds128(ws + r0 * 64 + ((c ^ sw0) << 4));
                const uint4 hi = lds128(ws + r1 * 64 + ((c ^ sw1) << 4));
                const uint32_t wl[4] = {lo.x, lo.y, lo.z, lo.w};
                const uint32_t wh[4] = {hi.x, hi.y, hi.z, hi.w};
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int ks = 2 * c + u;  // 32-k step within the stage
                    const uint32_t a0 = ternary4((wl[2 * u] >> sh) & 0x3333u);
                    const uint32_t a1 = ternary4((wh[2 * u] >> sh) & 0x3333u);
                    const uint32_t a2 = ternary4((wl[2 * u + 1] >> sh) & 0x3333u);
                    const uint32_t a3 = ternary4((wh[2 * u + 1] >> sh) & 0x3333u);
                    const uint8_t *box = as + (ks >> 2) * C::A_BOX;
                    const int ch = 2 * (ks & 3);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        const int tok = 8 * nt + g;
                        const uint8_t *rowp = box + tok * 128 + 4 * t;
                        const uint32_t b0 = lds32(rowp + ((ch ^ (tok & 7)) << 4));
                        const uint32_t b1 = lds32(rowp + (((ch + 1) ^ (tok & 7)) << 4));
                        mma_s8_16832(acc[nt], a0, a1, a2, a3, b0, b1);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
        // partial sums of this CTA: rows r0 / r1, tokens 8nt + 2t (+1)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int tk = 8 * nt + 2 * t;
            red[r0 * C::TOK + tk] = acc[nt][0];
            red[r0 * C::TOK + tk + 1] = acc[nt][1];
            red[r1 * C::TOK + tk] = acc[nt][2];
            red[r1 * C::TOK + tk + 1] = acc[nt][3];
        }
    }

    // ------------------------------------------------------------ split-K reduction + epilogue
    if (nsplit > 1) cluster_sync_all(); else __syncthreads();
    const int rlo = (int)(split * C::ROWS / nsplit), rhi = (int)((split + 1) * C::ROWS / nsplit);
    const int nr = rhi - rlo;
    const float a = *alpha;
    for (int o = threadIdx.x; o < nr * C::TOK; o += C::THREADS) {
        const int tok = o / nr, lr = rlo + o % nr;
        const int n = n0 + lr;
        int32_t sum = 0;
        if (nsplit > 1) {
            for (int q = 0; q < nsplit; ++q) sum += ld_dsmem_s32(&red[lr * C::TOK + tok], (uint32_t)q);
        } else {
            sum = red[lr * C::TOK + tok];
        }
        if (tok < M && n < N) {
            const float f = dequant_factor(a, __ldg(scale_x + tok), mode);
            out[(int64_t)tok * N + n] = __fmul_rn((float)sum, f);
            if (acc_out) acc_out[(int64_t)tok * N + n] = sum;
        }
    }
    if (nsplit > 1) cluster_sync_all();  // keep this CTA's partials alive for its peers
}

struct Plan {
    int warps, nsplit;
};

// Pick the cluster split so the CTA count fills whole waves of SMs.
Plan choose_plan(int N, int K, int sms) {
    const int nch = (K + 255) / 256;
    const int rowblocks = (N + 63) / 64;
    Plan best{4, 1};
    double best_score = -1.0;
    for (int ns = 1; ns <= 8 && ns <= nch; ++ns) {
        const long ctas = (long)rowblocks * ns;
        const long per_sm = (ctas + sms - 1) / sms;
        const double eff = (double)ctas / (double)(per_sm * sms);
        // prefer balance, then more CTAs in flight (up to ~4 per SM)
        const double score = eff + 0.01 * (per_sm <= 4 ? (double)per_sm : 0.0);
        if (score > best_score + 1e-9) {
            best_score = score;
            best = Plan{4, ns};
        }
    }
    return best;
}

template <int WARPS, int NT>
cudaError_t launch_cfg(const CUtensorMap &tw, const CUtensorMap &ta, const float *scale_x, int mode,
                       const float *alpha, int M, int N, int K, int nsplit, float *out, int32_t *acc_out,
                       bool pdl, cudaStream_t s) {
    using C = GemvCfg<WARPS, NT>;
    auto kern = gemv_kernel<WARPS, NT>;
    static bool done[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= kMaxDevices || !done[dev]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (e != cudaSuccess) return e;
        if (dev < kMaxDevices) done[dev] = true;
    }
    const int rowblocks = (N + C::ROWS - 1) / C::ROWS;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(rowblocks * nsplit));
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = s;
    cudaLaunchAttribute attrs[2];
    int na = 0;
    attrs[na].id = cudaLaunchAttributeClusterDimension;
    attrs[na].val.clusterDim.x = (unsigned)nsplit;
    attrs[na].val.clusterDim.y = 1;
    attrs[na].val.clusterDim.z = 1;
    ++na;
    if (pdl) {
        attrs[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attrs[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attrs;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, kern, tw, ta, scale_x, alpha, mode, M, N, K, nsplit, out, acc_out,
                              device_status_ptr());
}

}  // namespace

cudaError_t launch_gemv(const int8_t *codes, const float *scale_x, int mode, const uint8_t *packed,
                        const float *alpha, int M, int N, int K, float *out, int32_t *acc_out, bool pdl,
                        cudaStream_t s) {
    const Plan plan = choose_plan(N, K, sm_count());
    const int nt = M <= 8 ? 1 : 2;
    CUtensorMap tw, ta;
    if (!make_tmap_u8_2d(&tw, packed, (uint64_t)K / 4, (uint64_t)N, 64, 16 * plan.warps,
                         CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    if (!make_tmap_u8_2d(&ta, codes, (uint64_t)K, (uint64_t)M, 128, 8 * nt, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (nt == 1)
        return launch_cfg<4, 1>(tw, ta, scale_x, mode, alpha, M, N, K, plan.nsplit, out, acc_out, pdl, s);
    return launch_cfg<4, 2>(tw, ta, scale_x, mode, alpha, M, N, K, plan.nsplit, out, acc_out, pdl, s);
}

}  // namespace bitnet
