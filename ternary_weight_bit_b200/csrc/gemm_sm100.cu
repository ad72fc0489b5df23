// gemm_sm100.cu -- prefill path of steps 4b-5 on the 5th-generation tensor cores:
// tcgen05.mma kind::i8 (int8 x int8 -> int32) with the accumulators in TMEM.
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
// Per 128-k stage the shared memory carries only the activation tile (BT x 128 B)
// and the packed weights (128 x 32 B).
//
// Persistent: one CTA per SM walks the output tiles (weight-row block fastest, so
// an activation tile is reused from L2 by consecutive tiles).  Three rings keep the
// roles decoupled:
//   ST shared-memory stages  TMA -> unpack + MMA; freed by the MMA commit
//   AS TMEM weight slots     unpack -> MMA (32 columns = 128 k each); freed by the MMA commit
//   DB accumulator buffers   MMA -> epilogue; freed by the epilogue after tcgen05.ld
// With DB = 2 the epilogue of one tile overlaps the MMAs of the next; with DB = 1
// (BT = 256 fills TMEM) the MMAs of the next tile wait for the drain, while the
// TMA and unpack rings run on.
//
// Warp roles (64 + 128 UW + 128 threads):
//   warp 0       TMA producer; the whole warp runs the loop, an elected lane issues
//   warp 1       TMEM allocator and MMA issuer (4 x tcgen05.mma per stage, commits),
//                likewise warp-uniform with elected issue
//   UW sets of 4 unpack warps; set u takes the stages it with it % UW == u.  Warp w
//                owns TMEM lanes 32 (w % 4) .. +31 (= weight rows) of its slot.
//   4 epilogue warps: tcgen05.ld, out[m][n] = acc * f[m]; the fp32 (or bf16) tile goes
//                out through shared memory with one TMA bulk tensor store per 32 tokens.
//
// Split K (forward only, few output tiles): a work unit is (tile, split).  Two
// splits: the first to finish parks its int32 sums in the tile's output rows and
// raises a flag; the second, a CTA of this persistent grid, waits for the flag, adds
// and writes the output.  Four or eight: every split adds its sums into the zeroed
// output with integer atomics and the last one (per a tile counter) dequantises in
// place.  Both are exact, so the result equals the unsplit GEMM bit for bit.
// All waits are bounded; a timeout is recorded in the device status word.
#include <string.h>

#include "common.cuh"
#include "host.h"

namespace bitnet {

namespace {

constexpr int BW = 128;         // weight rows per tile (MMA M)
constexpr int BK = 128;         // k per stage
constexpr int OUT_TOKENS = 32;  // tokens per output store box

template <int BT_, int ST_, int AS_, int DB_, int UW_>
struct TcCfg {
    static constexpr int BT = BT_, ST = ST_, AS = AS_, DB = DB_, UW = UW_;
    static constexpr int THREADS = 64 + 128 * UW + 128;
    static constexpr int B_BYTES = BT * BK;      // activation tile
    static constexpr int P_BYTES = BW * BK / 4;  // packed weight tile (4 KB)
    static constexpr int B_OFF = 0;
    static constexpr int P_OFF = ST * B_BYTES;
    static constexpr int O_OFF = P_OFF + ST * P_BYTES;             // 2 x [32 tokens][128 rows] fp32 or bf16
    static constexpr int F_OFF = O_OFF + 2 * OUT_TOKENS * BW * 4;  // per-token dequant factors, DB rows
    static constexpr int BAR_OFF = F_OFF + DB * BT * 4;
    static constexpr int NUM_BARS = 2 * ST + 2 * AS + 2 * DB;
    static constexpr int TMEM_SLOT_OFF = BAR_OFF + NUM_BARS * 8;
    static constexpr int SMEM_USED = TMEM_SLOT_OFF + 16 + 1024;  // + alignment slack
    // At least 120 KB so that two CTAs never share an SM (each allocates all of TMEM).
    static constexpr int SMEM = SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t A_COL0 = DB * BT;  // D buffers first, then the weight slots
    static_assert(BT % 32 == 0 && BT >= 64 && BT <= 256, "MMA N");
    static_assert(DB * BT + 32 * AS <= 512, "TMEM budget");
    static_assert(SMEM_USED <= 232448, "shared memory budget");
    static_assert(UW <= ST && UW <= AS, "each unpack set advances by UW stages");
    static_assert(B_BYTES % 1024 == 0, "128B-swizzled tiles stay 1024-byte aligned");
    // D = s32, A = s8, B = s8, K-major both, N = BT, M = 128.
    static constexpr uint32_t IDESC = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BT >> 3) << 17) |
                                      ((uint32_t)(BW >> 4) << 24);
};

// The configurations the dispatcher chooses from.
using Cfg256 = TcCfg<256, 5, 4, 1, 2>;
using Cfg224 = TcCfg<224, 5, 2, 2, 2>;
using Cfg192 = TcCfg<192, 6, 4, 2, 2>;
using Cfg128 = TcCfg<128, 8, 8, 2, 2>;
using Cfg64 = TcCfg<64, 12, 8, 2, 2>;

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

// Tile t -> (weight-row block, token block); consecutive tiles walk the weight
// blocks of one token block, so the activation tile stays hot in L2.
struct TileMap {
    int nb_blocks;
    __device__ __forceinline__ void get(int t, int BT, int &n0, int &m0) const {
        n0 = (t % nb_blocks) * BW;
        m0 = (t / nb_blocks) * BT;
    }
};

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_act, const __grid_constant__ CUtensorMap tm_w,
               const __grid_constant__ CUtensorMap tm_out, int tma_out, const uint8_t *__restrict__ packed,
               const float *__restrict__ scale_x,
               const float *__restrict__ alpha, int mode, int M, int N, int K, void *__restrict__ out_v,
               int out_bf16, int32_t *__restrict__ acc_out, int splits, int *__restrict__ tile_cnt, int *status) {
    constexpr int BT = C::BT, ST = C::ST, AS = C::AS, DB = C::DB, UW = C::UW;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
    // barrier i at bar_base + 8 i: full[ST], sfree[ST], unpacked[AS], afree[AS], accfull[DB], accempty[DB]
    const uint32_t FULL = smem_u32(bars), SFREE = FULL + 8 * ST, UNPACKED = SFREE + 8 * ST,
                   AFREE = UNPACKED + 8 * AS, ACCFULL = AFREE + 8 * AS, ACCEMPTY = ACCFULL + 8 * DB;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::TMEM_SLOT_OFF);
    float *fac = reinterpret_cast<float *>(smem + C::F_OFF);
    __shared__ int s_last;  // split-K: this CTA added the last split of the tile
    const uint32_t sB0 = smem_u32(smem + C::B_OFF), sP0 = smem_u32(smem + C::P_OFF);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // Work unit u = (output tile u / splits, k-split u % splits); a split covers KBS
    // consecutive 128-k stages (splits divides K / 128).
    const int KBS = K / BK / splits;
    const TileMap tmap{(N + BW - 1) / BW};
    const int tiles = tmap.nb_blocks * ((M + BT - 1) / BT);
    const int units = tiles * splits;

    if (threadIdx.x == 0) {
        for (int i = 0; i < ST; ++i) {
            mbar_init(bars + i, 1);       // full: expect_tx arrival + TMA bytes
            mbar_init(bars + ST + i, 1);  // sfree: MMA commit
        }
        for (int i = 0; i < AS; ++i) {
            mbar_init(bars + 2 * ST + i, 4);       // unpacked: the four warps of one set
            mbar_init(bars + 2 * ST + AS + i, 1);  // afree: MMA commit
        }
        for (int i = 0; i < DB; ++i) {
            mbar_init(bars + 2 * ST + 2 * AS + i, 1);       // accfull: MMA commit
            mbar_init(bars + 2 * ST + 2 * AS + DB + i, 4);  // accempty: the four epilogue warps
        }
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
        }
        // Before the dependency wait only an L2 prefetch of the first tile's weight rows
        // (contiguous: 128 rows x K/4 bytes, at most 128 KB) is issued; every TMA load
        // follows the wait.
        if (lane == 0 && (int)blockIdx.x < units) {
            int n0, m0;
            tmap.get((int)blockIdx.x / splits, BT, n0, m0);
            const int nrows = (N - n0) < BW ? (N - n0) : BW;
            const uint32_t bytes = (uint32_t)nrows * (uint32_t)(K / 4);
            bulk_prefetch_l2(packed + (int64_t)n0 * (K / 4), bytes < (128u << 10) ? bytes : (128u << 10));
        }
        __syncwarp();
        pdl_launch_dependents();   // the next kernel may launch; it waits for this grid
        pdl_wait_prerequisites();  // activation codes come from the previous kernel
        bool ok = true, wrapped = false;
        int s = 0;
        uint32_t ph = 0;
        for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
            int n0, m0;
            tmap.get(u / splits, BT, n0, m0);
            const int kb0 = (u % splits) * KBS;
            for (int kb = kb0; kb < kb0 + KBS; ++kb) {
                if (wrapped && !mbar_wait_warp(SFREE + 8 * s, ph ^ 1u, status)) {
                    ok = false;
                    break;
                }
                mbar_expect_tx_elect(FULL + 8 * s, C::B_BYTES + C::P_BYTES);
                tma_load_2d_elect(sP0 + s * C::P_BYTES, &tm_w, FULL + 8 * s, kb * (BK / 4), n0);
                tma_load_2d_elect(sB0 + s * C::B_BYTES, &tm_act, FULL + 8 * s, kb * BK, m0);
                if (++s == ST) {
                    s = 0;
                    ph ^= 1u;
                    wrapped = true;
                }
            }
        }
        // every issued load must land before the CTA exits
        for (int i = 0; i < ST; ++i) {
            if (i < s) mbar_wait_warp(FULL + 8 * i, ph, status);
            else if (wrapped) mbar_wait_warp(FULL + 8 * i, ph ^ 1u, status);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        const uint64_t bdesc0 = smem_desc_sw128(sB0);
        int s = 0, a = 0, tc = 0;
        uint32_t ph = 0, aph = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++tc) {
            const int b = DB == 1 ? 0 : (tc & 1);
            // the epilogue must have drained this buffer (its previous use was unit tc - DB)
            if (tc >= DB && !mbar_wait_warp(ACCEMPTY + 8 * b, (uint32_t)((tc / DB) - 1) & 1u, status)) break;
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + (uint32_t)(b * BT);
            for (int kb = 0; kb < KBS; ++kb) {
                if (!mbar_wait_warp(FULL + 8 * s, ph, status) || !mbar_wait_warp(UNPACKED + 8 * a, aph, status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // the descriptor's start-address field advances by the stage offset / 16
                const uint64_t bdesc = bdesc0 + (uint64_t)((uint32_t)(s * C::B_BYTES) >> 4);
                const uint32_t a_tmem = tmem_base + C::A_COL0 + 32 * a;
#pragma unroll
                for (int j = 0; j < BK / 32; ++j)  // K = 32 per MMA: 8 TMEM columns of A, 32 bytes of B rows
                    umma_i8_ts_elect(d_tmem, a_tmem + 8 * j, bdesc + (uint64_t)(2 * j), C::IDESC,
                                     (kb | j) != 0 ? 1u : 0u);
                umma_commit_elect(SFREE + 8 * s);  // stage s (activation tile, packed weights) is free
                umma_commit_elect(AFREE + 8 * a);  // weight slot a is free
                if (++s == ST) {
                    s = 0;
                    ph ^= 1u;
                }
                if (++a == AS) {
                    a = 0;
                    aph ^= 1u;
                }
            }
            umma_commit_elect(ACCFULL + 8 * b);  // this tile's accumulator is complete
        }
    } else if (warp < 2 + 4 * UW) {
        // ------------------------------------------------------------ unpack into TMEM
        const int q = warp & 3;           // TMEM lane quarter of this warp
        const int set = (warp - 2) >> 2;  // takes the stages it with it % UW == set
        const int r = 32 * q + lane;      // weight row within the tile (= TMEM lane)
        const uint32_t lane_off = (uint32_t)(32 * q) << 16;
        const uint32_t sw = (uint32_t)((r >> 2) & 1) << 4;  // 32B swizzle of the packed row
        const uint32_t prow = sP0 + (uint32_t)r * 32;
        int s = set, a = set, turn = 0;
        uint32_t ph = 0, aph = 0;
        bool awrapped = false, ok = true;
        for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
            for (int kb = 0; kb < KBS; ++kb) {
                const bool mine = turn == set;
                if (++turn == UW) turn = 0;
                if (!mine) continue;
                if (!mbar_wait_u32(FULL + 8 * s, ph, status)) {
                    ok = false;
                    break;
                }
                const uint32_t bp = prow + s * C::P_BYTES;
                const uint4 p0 = lds128(bp + (0u ^ sw));
                const uint4 p1 = lds128(bp + (16u ^ sw));
                const uint32_t w[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
                uint32_t av[32];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint32_t s0 = w[c] & 0x33333333u;         // k = 16c + 0..7
                    const uint32_t s1 = (w[c] >> 2) & 0x33333333u;  // k = 16c + 8..15
                    av[4 * c + 0] = ternary4(s0);
                    av[4 * c + 1] = ternary4(s0 >> 16);
                    av[4 * c + 2] = ternary4(s1);
                    av[4 * c + 3] = ternary4(s1 >> 16);
                }
                // the slot's previous use was stage it - AS
                if (awrapped && !mbar_wait_u32(AFREE + 8 * a, aph ^ 1u, status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();  // order after the MMA that freed this slot
                tmem_st_32x32b_x32(tmem_base + lane_off + C::A_COL0 + 32 * a, av);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bars + 2 * ST + a);
                s += UW;
                if (s >= ST) {
                    s -= ST;
                    ph ^= 1u;
                }
                a += UW;
                if (a >= AS) {
                    a -= AS;
                    aph ^= 1u;
                    awrapped = true;
                }
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;
        const int r = 32 * q + lane;  // weight row within the tile (= TMEM lane)
        const uint32_t lane_off = (uint32_t)(32 * q) << 16;
        const int et = threadIdx.x - (64 + 128 * UW);  // 0..127
        float *obuf = reinterpret_cast<float *>(smem + C::O_OFF);
        const uint32_t sO0 = smem_u32(obuf);
        float *out = reinterpret_cast<float *>(out_v);                   // fp32 output (and split-K image)
        __nv_bfloat16 *outh = reinterpret_cast<__nv_bfloat16 *>(out_v);  // bf16 output (never split)
        const int obytes = out_bf16 ? 2 : 4;
        if (et == 0 && tma_out) tma_prefetch_desc(&tm_out);
        pdl_wait_prerequisites();
        const float a_scale = *alpha;
        int tc = 0, ck = 0;
        int32_t *acc_img = reinterpret_cast<int32_t *>(out);  // split-K: out holds int32 sums first
        for (int u = blockIdx.x; u < units; u += gridDim.x, ++tc) {
            const int b = DB == 1 ? 0 : (tc & 1);
            const int tile = u / splits;
            int n0, m0;
            tmap.get(tile, BT, n0, m0);
            for (int i = et; i < BT; i += 128) {
                const int m = m0 + i;
                fac[b * BT + i] = m < M ? dequant_factor(a_scale, __ldg(scale_x + m), mode) : 0.0f;
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (!mbar_wait_u32(ACCFULL + 8 * b, (uint32_t)(tc / DB) & 1u, status)) break;
            tc_fence_after();
            const int n = n0 + r;
            // Pair split (two halves of K): the first half to finish parks its int32 sums
            // in the tile's own output rows, the second adds them and writes the result.
            bool pair_first = false, pair_second = false;
            if (splits == 2) {
                if (et == 0) s_last = atomicAdd(tile_cnt + tile, 1);  // 0: first, 1: second
                asm volatile("bar.sync 1, 128;" ::: "memory");
                pair_second = s_last != 0;
                pair_first = !pair_second;
                if (pair_second) {
                    if (et == 0) flag_wait_set(tile_cnt + kPairFlags + tile, status);
                    asm volatile("bar.sync 1, 128;" ::: "memory");
                    __threadfence();
                }
            } else if (splits > 1) {
                // Add this split's partial sums to the int32 image of the tile (integer
                // atomics: the total does not depend on their order).
#pragma unroll 1
                for (int c = 0; c < BT / 32; ++c) {
                    if (m0 + 32 * c >= M) break;
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(tmem_base + lane_off + (uint32_t)(b * BT + 32 * c), v);
                    tmem_wait_ld();
                    if (n < N) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const int m = m0 + 32 * c + j;
                            if (m < M) atomicAdd(acc_img + (int64_t)m * N + n, (int)v[j]);
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bars + 2 * ST + 2 * AS + DB + b);  // the buffer may be overwritten
                __threadfence();  // this thread's additions are performed before the count below
                asm volatile("bar.sync 1, 128;" ::: "memory");
                if (et == 0) s_last = atomicAdd(tile_cnt + tile, 1) == splits - 1;
                asm volatile("bar.sync 1, 128;" ::: "memory");
                if (s_last) {
                    // the last split of this tile: dequantise the sums in place
                    __threadfence();
#pragma unroll 1
                    for (int c = 0; c < BT / 32; ++c) {
                        if (m0 + 32 * c >= M || n >= N) break;
                        int32_t sums[32];  // all 32 loads in flight before any use
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const int m = m0 + 32 * c + j;
                            sums[j] = m < M ? __ldcg(acc_img + (int64_t)m * N + n) : 0;
                        }
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const int m = m0 + 32 * c + j;
                            if (m < M) {
                                out[(int64_t)m * N + n] = __fmul_rn((float)sums[j], fac[b * BT + 32 * c + j]);
                                if (acc_out) acc_out[(int64_t)m * N + n] = sums[j];
                            }
                        }
                    }
                    if (et == 0) tile_cnt[tile] = 0;  // ready for the next call
                }
                asm volatile("bar.sync 1, 128;" ::: "memory");  // fac row b and s_last are reused
                continue;
            }
#pragma unroll 1
            for (int c = 0; c < BT / 32; ++c) {
                if (m0 + 32 * c >= M) break;  // the rest of the tile lies past the last token (uniform)
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem_base + lane_off + (uint32_t)(b * BT + 32 * c), v);
                tmem_wait_ld();
                if (splits == 2) {
                    // A whole 32-token chunk of a full-width tile is parked in a coalesced
                    // order: row r's 32 sums fill 128 contiguous bytes of token row
                    // m0 + 32c + r/4 at column n0 + 32 (r % 4).  Ragged chunks keep the
                    // natural [token][row] order.
                    const bool whole = m0 + 32 * c + 32 <= M && n0 + BW <= N && (N & 3) == 0;
                    int32_t *seg = acc_img + (int64_t)(m0 + 32 * c + (r >> 2)) * N + n0 + 32 * (r & 3);
                    if (pair_first) {
                        if (whole) {
#pragma unroll
                            for (int q4 = 0; q4 < 8; ++q4)
                                *reinterpret_cast<int4 *>(seg + 4 * q4) =
                                    make_int4((int)v[4 * q4], (int)v[4 * q4 + 1], (int)v[4 * q4 + 2], (int)v[4 * q4 + 3]);
                        } else if (n < N) {
#pragma unroll
                            for (int j = 0; j < 32; ++j) {
                                const int m = m0 + 32 * c + j;
                                if (m < M) acc_img[(int64_t)m * N + n] = (int)v[j];
                            }
                        }
                        continue;  // the second half writes the output
                    }
                    if (whole) {
                        int4 pq[8];
#pragma unroll
                        for (int q4 = 0; q4 < 8; ++q4) pq[q4] = __ldcg(reinterpret_cast<const int4 *>(seg + 4 * q4));
#pragma unroll
                        for (int q4 = 0; q4 < 8; ++q4) {
                            v[4 * q4] = (uint32_t)((int)v[4 * q4] + pq[q4].x);
                            v[4 * q4 + 1] = (uint32_t)((int)v[4 * q4 + 1] + pq[q4].y);
                            v[4 * q4 + 2] = (uint32_t)((int)v[4 * q4 + 2] + pq[q4].z);
                            v[4 * q4 + 3] = (uint32_t)((int)v[4 * q4 + 3] + pq[q4].w);
                        }
                    } else if (n < N) {
                        int32_t pq[32];
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const int m = m0 + 32 * c + j;
                            pq[j] = m < M ? __ldcg(acc_img + (int64_t)m * N + n) : 0;
                        }
#pragma unroll
                        for (int j = 0; j < 32; ++j) v[j] = (uint32_t)((int)v[j] + pq[j]);
                    }
                    // every thread's reads of the parked sums are done before any output
                    // of this chunk replaces them
                    asm volatile("bar.sync 1, 128;" ::: "memory");
                }
                if (tma_out) {
                    // [32 tokens][128 rows] through shared memory, one bulk tensor store
                    const int buf = ck & 1;
                    if (et == 0 && ck >= 2) bulk_wait_group_read<1>();  // the store that read buf is done
                    asm volatile("bar.sync 1, 128;" ::: "memory");
                    if (out_bf16) {
                        __nv_bfloat16 *sb = reinterpret_cast<__nv_bfloat16 *>(obuf) + buf * (OUT_TOKENS * BW);
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            sb[j * BW + r] = __float2bfloat16_rn(__fmul_rn((float)(int)v[j], fac[b * BT + 32 * c + j]));
                    } else {
                        float *sb = obuf + buf * (OUT_TOKENS * BW);
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            sb[j * BW + r] = __fmul_rn((float)(int)v[j], fac[b * BT + 32 * c + j]);
                    }
                    fence_proxy_async_smem();
                    asm volatile("bar.sync 1, 128;" ::: "memory");
                    if (et == 0) {
                        tma_store_2d(&tm_out, sO0 + (uint32_t)(buf * OUT_TOKENS * BW * obytes), n0, m0 + 32 * c);
                        bulk_commit_group();
                    }
                    ++ck;
                } else if (n < N) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int m = m0 + 32 * c + j;
                        if (m >= M) continue;
                        const float y = __fmul_rn((float)(int)v[j], fac[b * BT + 32 * c + j]);
                        if (out_bf16) outh[(int64_t)m * N + n] = __float2bfloat16_rn(y);
                        else out[(int64_t)m * N + n] = y;
                    }
                }
                if (acc_out && n < N) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int m = m0 + 32 * c + j;
                        if (m < M) acc_out[(int64_t)m * N + n] = (int)v[j];
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bars + 2 * ST + 2 * AS + DB + b);  // the buffer may be overwritten
            if (pair_first) {
                __threadfence();  // this thread's parked sums are visible before the flag below
                asm volatile("bar.sync 1, 128;" ::: "memory");
                if (et == 0) atomicExch(tile_cnt + kPairFlags + tile, 1);
            } else if (pair_second && et == 0) {
                tile_cnt[tile] = 0;  // ready for the next call
                tile_cnt[kPairFlags + tile] = 0;
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");              // fac row b is rewritten DB tiles later
        }
        if (et == 0 && tma_out) bulk_wait_group<0>();  // the last stores have landed
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

template <class C>
cudaError_t launch_cfg(const int8_t *codes, const float *scale_x, int mode, const uint8_t *packed,
                       const float *alpha, int M, int N, int K, void *out, bool out_bf16, int32_t *acc_out,
                       int splits, int *tile_cnt, bool pdl, cudaStream_t s) {
    CUtensorMap ta, tw, to;
    if (!make_tmap_u8_2d(&ta, codes, (uint64_t)K, (uint64_t)M, BK, C::BT, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (!make_tmap_u8_2d(&tw, packed, (uint64_t)K / 4, (uint64_t)N, BK / 4, BW, CU_TENSOR_MAP_SWIZZLE_32B))
        return cudaErrorInvalidValue;
    // The bulk-store epilogue needs a 16-byte row pitch and base, and a box that fits.
    memset(&to, 0, sizeof(to));
    // (N elements of 4 or 2 bytes per row: N % 4 == 0 for fp32, N % 8 == 0 for bf16)
    const bool store_ok = splits <= 2 && N % (out_bf16 ? 8 : 4) == 0 && M >= OUT_TOKENS && N >= BW &&
                          (reinterpret_cast<uintptr_t>(out) & 15) == 0;
    const int tma_out =
        store_ok && make_tmap_out_2d(&to, out, out_bf16, (uint64_t)N, (uint64_t)M, BW, OUT_TOKENS) ? 1 : 0;
    auto kern = gemm_tc_kernel<C>;
    static bool done[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= kMaxDevices || !done[dev]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (e != cudaSuccess) return e;
        if (dev < kMaxDevices) done[dev] = true;
    }
    const long units = (long)((N + BW - 1) / BW) * ((M + C::BT - 1) / C::BT) * splits;
    const int grid = (int)(units < sm_count() ? units : sm_count());
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = s;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, ta, tw, to, tma_out, packed, scale_x, alpha, mode, M, N, K, out,
                              out_bf16 ? 1 : 0, acc_out, splits, tile_cnt, device_status_ptr());
}

}  // namespace

// Modelled time of a (token tile, k-split) choice, in units of one 128-k stage of one
// tile: rounds of work units per SM x (stages per unit x relative stage cost + a
// drain stall per unit when the accumulator is single-buffered + the split fixup).
// All constants are B200 measurements: a stage takes about as long at 192..256
// tokens; the single-buffered 256-token tile stalls about 10 stages per tile; a tile
// split in two costs about 5 BT / 16 stages more (the first half parks its sums, the
// second reads them back chunk by chunk), one split further with atomics about
// 20 + BT / 4, so splitting only pays for few output tiles and long K.
double gemm_tile_cost(int bt, int splits, int M, int N, int K, int sms) {
    const double w = bt >= 192 ? 1.0 : (bt >= 128 ? 0.93 : 0.81);
    const double drain = bt == 256 ? 10.0 : 0.0;
    const double split_cost = splits == 1 ? 0.0 : (splits == 2 ? bt * 5.0 / 16.0 : 20.0 + bt / 4.0);
    const long units = (long)((N + BW - 1) / BW) * ((M + bt - 1) / bt) * splits;
    const long rounds = (units + sms - 1) / sms;
    return (double)rounds * ((double)(K / BK / splits) * w + drain + split_cost);
}

namespace {
int g_forced_tile = 0;    // 0: automatic
int g_forced_splits = 0;  // 0: automatic
}  // namespace

bool gemm_force_tile(int bt) {
    if (bt != 0 && bt != 256 && bt != 224 && bt != 192 && bt != 128 && bt != 64) return false;
    g_forced_tile = bt;
    return true;
}

bool gemm_force_splits(int splits) {
    if (splits != 0 && splits != 1 && splits != 2 && splits != 4 && splits != 8) return false;
    g_forced_splits = splits;
    return true;
}

GemmPlan gemm_plan(int M, int N, int K, int sms, int max_split_tiles) {
    static const int tiles_c[] = {256, 224, 192, 128, 64};
    static const int splits_c[] = {1, 2, 4, 8};
    GemmPlan best{256, 1};
    double best_cost = 1e300;
    const int KB = K / BK;
    // a forced split count applies where splitting is allowed at all (the forward) and
    // the shape admits it; otherwise the automatic choice stands
    for (int pass = (g_forced_splits && max_split_tiles > 0) ? 0 : 1; pass < 2 && best_cost == 1e300; ++pass) {
        for (int bt : tiles_c) {
            if (g_forced_tile && bt != g_forced_tile) continue;
            const long tiles = (long)((N + BW - 1) / BW) * ((M + bt - 1) / bt);
            for (int sp : splits_c) {
                if (pass == 0 && sp != g_forced_splits) continue;
                if (sp > 1 && (tiles > max_split_tiles || KB % sp != 0 || KB / sp < 4)) continue;
                if (sp == 2 && tiles > kPairFlags) continue;  // arrival counters and flags share the workspace
                const double c = gemm_tile_cost(bt, sp, M, N, K, sms);
                if (c < best_cost * 0.999) {
                    best = GemmPlan{bt, sp};
                    best_cost = c;
                }
            }
        }
    }
    return best;
}

int gemm_pick_tile(int M, int N, int K, int sms) { return gemm_plan(M, N, K, sms, 0).token_tile; }

cudaError_t launch_gemm_tc(const int8_t *codes, const float *scale_x, int mode, const uint8_t *packed,
                           const float *alpha, int M, int N, int K, void *out, int32_t *acc_out, bool pdl,
                           cudaStream_t s, GemmPlan plan, int *tile_cnt, bool out_bf16) {
    if (plan.token_tile == 0) plan = gemm_plan(M, N, K, sm_count(), 0);
    const int sp = plan.splits;
    // a split GEMM accumulates int32 in the output itself, which a bf16 output cannot hold
    if (sp < 1 || (sp > 1 && (!tile_cnt || (K / BK) % sp != 0 || out_bf16))) return cudaErrorInvalidValue;
    switch (plan.token_tile) {
    case 256: return launch_cfg<Cfg256>(codes, scale_x, mode, packed, alpha, M, N, K, out, out_bf16, acc_out, sp, tile_cnt, pdl, s);
    case 224: return launch_cfg<Cfg224>(codes, scale_x, mode, packed, alpha, M, N, K, out, out_bf16, acc_out, sp, tile_cnt, pdl, s);
    case 192: return launch_cfg<Cfg192>(codes, scale_x, mode, packed, alpha, M, N, K, out, out_bf16, acc_out, sp, tile_cnt, pdl, s);
    case 128: return launch_cfg<Cfg128>(codes, scale_x, mode, packed, alpha, M, N, K, out, out_bf16, acc_out, sp, tile_cnt, pdl, s);
    case 64: return launch_cfg<Cfg64>(codes, scale_x, mode, packed, alpha, M, N, K, out, out_bf16, acc_out, sp, tile_cnt, pdl, s);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace bitnet
