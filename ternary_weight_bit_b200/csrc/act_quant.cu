// act_quant.cu -- steps 1-3 of the H-BitLinear forward, fused: per-token RMSNorm,
// optional Fast Walsh-Hadamard transform, int8-absmax / int4-absmean quantisation.
//
// Method: bitnet_v2_engine.py page -- HBitLinear.forward (normalise, rotate,
// quantise), fast_hadamard_transform and Eq. 3/4 (H_m = (1/sqrt2)[[H,H],[H,-H]]),
// quantize_act_int8 (Eq. 5) and quantize_act_int4 (Eq. 6).
//
// X is read from HBM exactly once and the codes are written once; everything in
// between stays on chip.  Few tokens: one CTA per token (the plain and the per-token
// FWHT kernels).  Many tokens with 2^11 <= K <= 2^14: the streaming FWHT kernel, a
// persistent grid that takes the tokens in turn (described at its definition).
//
// Per-token FWHT kernel (K = 2^LOGK): each thread owns E = 2^ELOG elements.  The transform
// runs as unnormalised radix-2 butterflies (a+b, a-b) over bits 0, 1, ..., LOGK-1
// in increasing order, in phases of ELOG bits: inside a phase the butterflies are
// in registers; between phases the token is transposed through shared memory so
// that the next ELOG index bits become register bits.  The 1/sqrt2 per stage is
// folded into one multiplier 2^(-LOGK/2) applied together with the RMSNorm factor
// (exact for even LOGK).  This reorders the roundings of the page's per-stage
// scaling; results differ from it only in the last bits.
#include "common.cuh"
#include "host.h"

namespace bitnet {

namespace {

// ------------------------------------------------------------------ reductions
template <int T>
__device__ __forceinline__ float block_sum(float v, float *red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    constexpr int W = T / 32;
    if constexpr (W == 1) {
        return v;
    } else {
        const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
        __syncthreads();  // red may still be read from a previous reduction
        if (lane == 0) red[warp] = v;
        __syncthreads();
        float s = lane < W ? red[lane] : 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        return s;
    }
}

template <int T>
__device__ __forceinline__ float block_max(float v, float *red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    constexpr int W = T / 32;
    if constexpr (W == 1) {
        return v;
    } else {
        const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
        __syncthreads();
        if (lane == 0) red[warp] = v;
        __syncthreads();
        float s = lane < W ? red[lane] : 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s = fmaxf(s, __shfl_xor_sync(0xffffffffu, s, o));
        return s;
    }
}

// ------------------------------------------------------------------ quantiser
// Round-clip y*s to [lo, hi] with round-half-to-even in one fused multiply-add:
// y*s + 1.5*2^23, rounded once, is 1.5*2^23 plus the integer nearest the exact product
// (ties to even) while |y*s| < 2^22, that integer sitting in the low mantissa bits.
// The clip acts on the biased value (an integer in [lo, hi] then), which also holds any
// larger |y*s| at the bound.  Returns the whole word (code in the low byte); clips only
// when asked.  Against rounding the product first, the code can change only where the
// exact product lies within half an ulp of a rounding tie.
__device__ __forceinline__ uint32_t quant_bits(float y, float s, float lo, float hi, bool clip) {
    constexpr float kBias = 12582912.0f;  // 1.5 * 2^23
    float v = __fmaf_rn(y, s, kBias);
    if (clip) v = fminf(fmaxf(v, kBias + lo), kBias + hi);
    return __float_as_uint(v);
}

// Low bytes of four words -> one word (byte permutes).
__device__ __forceinline__ uint32_t pack4_perm(uint32_t f0, uint32_t f1, uint32_t f2, uint32_t f3) {
    return __byte_perm(__byte_perm(f0, f1, 0x0040), __byte_perm(f2, f3, 0x0040), 0x5410);
}

struct QuantParams {
    float s, lo, hi;
};

__device__ __forceinline__ QuantParams quant_params(float stat, float eps, int mode) {
    QuantParams q;
    if (mode == BITNET_ACT_INT8_ABSMAX) {
        q.s = __fdiv_rn(127.0f, __fadd_rn(stat, eps));
        q.lo = -128.0f;
        q.hi = 127.0f;
    } else {
        q.s = __fdiv_rn(2.64575131106459059f, __fadd_rn(stat, eps));
        q.lo = -8.0f;
        q.hi = 7.0f;
    }
    return q;
}

__device__ __forceinline__ float rms_factor(float ss, int K, float eps) {
    return __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(ss, (float)K), eps)));
}

// Load 8 consecutive elements (fp32 or bf16) starting at element index `idx`.
template <bool BF16>
__device__ __forceinline__ void load8(const void *X, int64_t idx, float *v) {
    if constexpr (BF16) {
        const uint4 u = __ldg(reinterpret_cast<const uint4 *>(reinterpret_cast<const uint16_t *>(X) + idx));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    } else {
        const float4 *p = reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(X) + idx);
        const float4 a = __ldg(p), b = __ldg(p + 1);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
}

template <bool BF16>
__device__ __forceinline__ float load1(const void *X, int64_t idx) {
    if constexpr (BF16)
        return __uint_as_float((uint32_t)__ldg(reinterpret_cast<const unsigned short *>(X) + idx) << 16);
    else
        return __ldg(reinterpret_cast<const float *>(X) + idx);
}

template <bool BF16>
__device__ __forceinline__ void load4(const void *X, int64_t idx, float *v) {
    if constexpr (BF16) {
        const uint2 u = __ldg(reinterpret_cast<const uint2 *>(reinterpret_cast<const uint16_t *>(X) + idx));
        v[0] = __uint_as_float(u.x << 16);
        v[1] = __uint_as_float(u.x & 0xFFFF0000u);
        v[2] = __uint_as_float(u.y << 16);
        v[3] = __uint_as_float(u.y & 0xFFFF0000u);
    } else {
        const float4 a = __ldg(reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(X) + idx));
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    }
}

// ------------------------------------------------------------------ input sources
// The kernels read their per-token input through a source: XSrc reads X itself;
// SwigluSrc forms the SwiGLU product silu(gate) * up of a BitNet v2 FFN on the fly
// (bitnet_v2_engine.py page, BitNetV2FFN.forward: F.silu(gate_proj(x)) * up_proj(x)),
// so the intermediate activation never makes an fp32 round trip through HBM.
template <bool BF16>
struct XSrc {
    const void *X;
    __device__ __forceinline__ void get8(int64_t idx, float *v) const { load8<BF16>(X, idx, v); }
    __device__ __forceinline__ void get4(int64_t idx, float *v) const { load4<BF16>(X, idx, v); }
    __device__ __forceinline__ float get1(int64_t idx) const { return load1<BF16>(X, idx); }
    // L2 prefetch of n elements from idx (a hint: it returns no data, so it is safe before
    // the dependency wait -- L2 is where every write lands, so what is read later is current)
    __device__ __forceinline__ void prefetch(int64_t idx, int n) const {
        bulk_prefetch_l2(reinterpret_cast<const uint8_t *>(X) + idx * (BF16 ? 2 : 4), (uint32_t)n * (BF16 ? 2 : 4));
    }
};

// silu(g) * u with silu(g) = g / (1 + e^-g), each step one IEEE rounding.
__device__ __forceinline__ float swiglu(float g, float u) {
    return __fmul_rn(__fdiv_rn(g, __fadd_rn(1.0f, expf(-g))), u);
}

template <bool BF16>
struct SwigluSrc {
    const void *gate, *up;
    __device__ __forceinline__ void prefetch(int64_t idx, int n) const {
        bulk_prefetch_l2(reinterpret_cast<const uint8_t *>(gate) + idx * (BF16 ? 2 : 4), (uint32_t)n * (BF16 ? 2 : 4));
        bulk_prefetch_l2(reinterpret_cast<const uint8_t *>(up) + idx * (BF16 ? 2 : 4), (uint32_t)n * (BF16 ? 2 : 4));
    }
    __device__ __forceinline__ void get8(int64_t idx, float *v) const {
        float u[8];
        load8<BF16>(gate, idx, v);
        load8<BF16>(up, idx, u);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = swiglu(v[i], u[i]);
    }
    __device__ __forceinline__ void get4(int64_t idx, float *v) const {
        float u[4];
        load4<BF16>(gate, idx, v);
        load4<BF16>(up, idx, u);
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = swiglu(v[i], u[i]);
    }
};

// ------------------------------------------------------------------ FWHT kernel
template <int LOGK>
struct FwhtShape {
    static constexpr int K = 1 << LOGK;
    static constexpr int ELOG = (LOGK - 5) < 5 ? (LOGK - 5) : 5;  // elements per thread = 2^ELOG
    static constexpr int E = 1 << ELOG;
    static constexpr int T = K / E;  // threads per CTA (>= 32)
    static constexpr int PHASES = (LOGK + ELOG - 1) / ELOG;
};

// Index of register r of thread tid in phase p is tid_part(p, tid) | reg_part(p, r):
// the register bits are [lo, lo+nb) plus, in a short last phase, the low `pass`
// bits as passengers; the thread bits fill the rest.  The two parts occupy
// disjoint bits, so their padded addresses add up (see pad()).
template <int LOGK, int ELOG>
__device__ __forceinline__ int tid_part(int p, int tid) {
    const int lo = p * ELOG;
    const int nb = (LOGK - lo) < ELOG ? (LOGK - lo) : ELOG;
    const int pass = ELOG - nb;
    const int tl = lo - pass;
    return ((tid & ((1 << tl) - 1)) << pass) | ((tid >> tl) << (lo + nb));
}
template <int LOGK, int ELOG>
__device__ __forceinline__ int reg_part(int p, int r) {
    const int lo = p * ELOG;
    const int nb = (LOGK - lo) < ELOG ? (LOGK - lo) : ELOG;
    const int pass = ELOG - nb;
    return (r & ((1 << pass) - 1)) | ((r >> pass) << lo);
}

// Shared-memory position of element i: one pad word after every 32 elements
// spreads the strided phase accesses over the banks.  For disjoint bit fields
// a, b: pad(a | b) = pad(a) + pad(b), so every register's address is a
// compile-time offset from one per-thread base.
__device__ __forceinline__ int pad(int i) { return i + (i >> 5); }

// Zero the token's row of a following split-K GEMM's output (it adds int32 partial
// sums there; a two-way split needs no zero rows) and, in CTA 0, that GEMM's tile
// counters.  Runs after the dependency
// wait: the buffers may still be read by earlier kernels until then.
__device__ __forceinline__ void zero_fill(const ZeroFill &z, int64_t token) {
    if (z.rows) {
        uint32_t *row = z.rows + token * z.row_words;
        for (int i = threadIdx.x; i < z.row_words; i += blockDim.x) row[i] = 0u;
    }
    if (token == 0 && z.cnt)
        for (int i = threadIdx.x; i < z.cnt_n; i += blockDim.x) z.cnt[i] = 0;
}

// Per-token scalars shared through shared memory after a token's reduction.
struct FwhtScalars {
    float s_eff, stat;
};

// The FWHT and quantiser for one token whose phase-0 values are in v (thread tid owns
// elements [tid*E, tid*E + E)); ss is this thread's partial sum of x^2.  Gain, log2 K
// butterfly stages in phases of ELOG bits with shared-memory transposes between them,
// then ONE block reduction of (sum x^2, max|z| or sum|z|) over the unscaled transform z:
// RMSNorm's factor r and the 2^(-m/2) of the m stages are one scalar rho that commutes
// with the transform, so y = rho z, gamma = rho max|z| (exact: rounding is monotone) or
// beta = rho sum|z| / K, and the code is rne(z * (rho s)) -- the same values as scaling
// first, up to the rounding of one product.  `hook` runs once every thread has read its
// phase-0 values and passed the first transpose (the streaming kernel refills its input
// buffer there).  Barriers: the first transpose needs none before its writes -- every
// thread's previous reads of sm, red and sc were followed by this call's or the previous
// call's reduction barriers.
template <int LOGK, class Hook>
__device__ __forceinline__ void fwht_quant_token(float (&v)[FwhtShape<LOGK>::E], float ss, int64_t token,
                                                 const float *__restrict__ gain, float eps, int mode,
                                                 int8_t *__restrict__ codes, float *__restrict__ scale_x, float *sm,
                                                 float2 *red, FwhtScalars *sc, Hook hook) {
    using S = FwhtShape<LOGK>;
    constexpr int K = S::K, ELOG = S::ELOG, E = S::E, T = S::T, P = S::PHASES;
    constexpr int W = T / 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t row = token * K;
    // Materialise the partial sum now: left to itself the compiler sinks its products
    // to the reduction at the end and keeps the E inputs alive through the transform.
    asm volatile("" : "+f"(ss));

    if (gain != nullptr) {
#pragma unroll
        for (int r = 0; r < E; ++r) v[r] = __fmul_rn(v[r], __ldg(gain + tid * E + r));
    }

    // Butterflies over all LOGK bits, in increasing bit order.
#pragma unroll
    for (int p = 0; p < P; ++p) {
        if (p > 0) {
            if (p > 1) __syncthreads();  // every thread has read the previous phase's layout
            float *wb = sm + pad(tid_part<LOGK, ELOG>(p - 1, tid));
#pragma unroll
            for (int r = 0; r < E; ++r) wb[pad(reg_part<LOGK, ELOG>(p - 1, r))] = v[r];
            __syncthreads();
            if (p == 1) hook();
            const float *rb = sm + pad(tid_part<LOGK, ELOG>(p, tid));
#pragma unroll
            for (int r = 0; r < E; ++r) v[r] = rb[pad(reg_part<LOGK, ELOG>(p, r))];
        } else if (P == 1) {
            hook();
        }
        const int lo = p * ELOG;
        const int nb = (LOGK - lo) < ELOG ? (LOGK - lo) : ELOG;
        const int pass = ELOG - nb;
#pragma unroll
        for (int b = 0; b < ELOG; ++b) {
            if (b >= pass) {
                const int h = 1 << b;
#pragma unroll
                for (int r = 0; r < E; ++r) {
                    if ((r & h) == 0) {
                        const float a = v[r], c = v[r | h];
                        v[r] = __fadd_rn(a, c);
                        v[r | h] = __fsub_rn(a, c);
                    }
                }
            }
        }
    }

    // one reduction: (sum x^2, max|z| or sum|z|)
    const bool mean = mode != BITNET_ACT_INT8_ABSMAX;
    float st = 0.0f;
    if (mean) {
#pragma unroll
        for (int r = 0; r < E; ++r) st += fabsf(v[r]);
    } else {
#pragma unroll
        for (int r = 0; r < E; ++r) st = fmaxf(st, fabsf(v[r]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        ss += __shfl_xor_sync(0xffffffffu, ss, o);
        const float x = __shfl_xor_sync(0xffffffffu, st, o);
        st = mean ? st + x : fmaxf(st, x);
    }
    if constexpr (W > 1) {
        if (lane == 0) red[warp] = make_float2(ss, st);
        __syncthreads();
        if (warp == 0) {
            float2 q = lane < W ? red[lane] : make_float2(0.0f, 0.0f);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                q.x += __shfl_xor_sync(0xffffffffu, q.x, o);
                const float x = __shfl_xor_sync(0xffffffffu, q.y, o);
                q.y = mean ? q.y + x : fmaxf(q.y, x);
            }
            ss = q.x;
            st = q.y;
        }
    }
    if (tid == 0) {
        const float p2 = __int_as_float((127 - LOGK / 2) << 23);  // 2^(-floor(LOGK/2)), exact
        const float hs = (LOGK & 1) ? __fmul_rn(0.70710678118654752f, p2) : p2;
        const float rho = __fmul_rn(rms_factor(ss, K, eps), hs);
        const float rs = __fmul_rn(rho, st);
        const float stat = mean ? __fdiv_rn(rs, (float)K) : rs;
        const QuantParams qp = quant_params(stat, eps, mode);
        sc->s_eff = __fmul_rn(rho, qp.s);
        sc->stat = stat;
        scale_x[token] = stat;
    }
    __syncthreads();
    const float s_eff = sc->s_eff;
    const float lo = mean ? -8.0f : -128.0f, hi = mean ? 7.0f : 127.0f;
    // int8: |z s_eff| <= 127 (1 + 4u) < 127.5, so the clip can never act.

    // Store the codes in the last phase's layout.
    constexpr int LASTLO = (P - 1) * ELOG;
    constexpr int LASTNB = (LOGK - LASTLO) < ELOG ? (LOGK - LASTLO) : ELOG;
    constexpr int LASTPASS = ELOG - LASTNB;
    int8_t *out = codes + row + tid_part<LOGK, ELOG>(P - 1, tid);
    if constexpr (LASTPASS >= 2) {
#pragma unroll
        for (int r = 0; r < E; r += 4) {
            uint32_t f[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) f[e] = quant_bits(v[r + e], s_eff, lo, hi, mean);
            *reinterpret_cast<uint32_t *>(out + reg_part<LOGK, ELOG>(P - 1, r)) = pack4_perm(f[0], f[1], f[2], f[3]);
        }
    } else {
#pragma unroll
        for (int r = 0; r < E; ++r)
            out[reg_part<LOGK, ELOG>(P - 1, r)] = (int8_t)(quant_bits(v[r], s_eff, lo, hi, mean) & 0xFFu);
    }
}

struct NoHook {
    __device__ __forceinline__ void operator()() const {}
};

template <int LOGK, class Src>
__global__ void __launch_bounds__(FwhtShape<LOGK>::T)
act_quant_fwht_kernel(Src src, const float *__restrict__ gain, float eps, int mode,
                      int8_t *__restrict__ codes, float *__restrict__ scale_x, ZeroFill zf) {
    using S = FwhtShape<LOGK>;
    constexpr int K = S::K, E = S::E;
    extern __shared__ __align__(16) float sm[];  // K + K/32 floats (padded)
    __shared__ float2 red[32];
    __shared__ FwhtScalars sc;

    // Let the GEMM launch now and start streaming its weights; then wait for X, which
    // may come from the previous kernel.  The GEMM waits for this kernel before it
    // reads the codes, so the order of the data is kept.
    pdl_launch_dependents();
    if (threadIdx.x == 0) src.prefetch((int64_t)blockIdx.x * K, K);  // warm L2 while the producer finishes
    pdl_wait_prerequisites();
    zero_fill(zf, blockIdx.x);

    const int tid = threadIdx.x;
    const int64_t row = (int64_t)blockIdx.x * K;
    float v[E];

    // Phase 0 layout: thread tid owns the E contiguous elements [tid*E, tid*E + E).
    if constexpr (E >= 8) {
#pragma unroll
        for (int c = 0; c < E / 8; ++c) src.get8(row + tid * E + 8 * c, v + 8 * c);
    } else {
        src.get4(row + tid * E, v);
    }

    float ss = 0.0f;
#pragma unroll
    for (int r = 0; r < E; ++r) ss = fmaf(v[r], v[r], ss);
    fwht_quant_token<LOGK>(v, ss, blockIdx.x, gain, eps, mode, codes, scale_x, sm, red, &sc, NoHook{});
}

// ------------------------------------------------------------------ streaming FWHT kernel
// For many tokens with 2^11 <= K <= 2^14: a persistent grid whose CTAs loop over tokens
// (t = blockIdx.x, + gridDim.x, ...), several CTAs resident per SM.  The transform takes
// two register phases and one shared-memory transpose.  With ELOG = ceil(LOGK/2)
// register bits and TLOG = LOGK - ELOG thread bits per phase:
//   phase 0: thread t holds elements t + (r << TLOG), r < 2^ELOG, so each load
//            instruction of a warp reads 32 consecutive elements, and runs the
//            butterflies of element bits TLOG..LOGK-1;
//   phase 1: thread t holds the 2^ELOG consecutive elements t*2^ELOG + r, read back as
//            16-byte units, and runs the butterflies of bits 0..TLOG-1 (for odd LOGK,
//            bit TLOG rides along untouched); its codes leave as 16-byte stores.
// Element i sits in shared memory at word i ^ (((i >> ELOG) & 7) << 2): the 16-byte unit
// index is XORed with three bits of the element's phase-1 owner, which keeps both the
// phase-0 word stores and the phase-1 16-byte loads free of bank conflicts.  The
// butterflies run on register pairs with the packed fp32 add and fma of sm_100 (a - b as
// fma(b, -1, a): the same single rounding as a subtraction), except in the register bit
// that forms the pairs.  The bits are transformed in another order than in the per-token
// kernel, so results differ from it in the last bits only.  Each token's row is prefetched
// into L2 one token ahead; the barriers per token are two: after the transpose's stores,
// and in the statistic's reduction, whose result every thread then finishes itself.
template <int LOGK>
struct StreamShape {
    static constexpr int K = 1 << LOGK;
    static constexpr int ELOG = (LOGK + 1) / 2;
    static constexpr int E = 1 << ELOG;       // elements per thread
    static constexpr int TLOG = LOGK - ELOG;
    static constexpr int T = 1 << TLOG;       // threads per CTA
    static constexpr int W = T / 32;
    static constexpr int MINB = (E >= 128 ? 384 : 512) / T;  // CTAs per SM the registers allow
    static constexpr int SMEM = K * 4;
};

// Butterflies of register bit b over E values held as E/2 pairs (pair j = registers 2j, 2j+1).
template <int NP>
__device__ __forceinline__ void butterfly_pairs(float2 (&v)[NP], int b) {
    if (b == 0) {
#pragma unroll
        for (int j = 0; j < NP; ++j) {
            const float a = v[j].x, c = v[j].y;
            v[j] = make_float2(__fadd_rn(a, c), __fsub_rn(a, c));
        }
    } else {
        const int h = 1 << (b - 1);
#pragma unroll
        for (int j = 0; j < NP; ++j) {
            if ((j & h) == 0) {
                const float2 a = v[j], c = v[j | h];
                v[j] = __fadd2_rn(a, c);
                v[j | h] = __ffma2_rn(c, make_float2(-1.0f, -1.0f), a);
            }
        }
    }
}

template <int LOGK, class Src>
__global__ void __launch_bounds__(StreamShape<LOGK>::T, StreamShape<LOGK>::MINB)
act_quant_fwht_stream_kernel(Src src, const float *__restrict__ gain, float eps, int mode, int64_t M,
                             int8_t *__restrict__ codes, float *__restrict__ scale_x, ZeroFill zf) {
    using S = StreamShape<LOGK>;
    constexpr int K = S::K, E = S::E, NP = E / 2, ELOG = S::ELOG, TLOG = S::TLOG, W = S::W;
    extern __shared__ __align__(16) float buf[];  // K floats, swizzled
    __shared__ float2 red[W];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool mean = mode != BITNET_ACT_INT8_ABSMAX;
    constexpr float kBias = 12582912.0f;  // 1.5 * 2^23, see quant_bits
    const float qlo = kBias + (mean ? -8.0f : -128.0f), qhi = kBias + (mean ? 7.0f : 127.0f);
    const float p2 = __int_as_float((127 - LOGK / 2) << 23);  // 2^(-floor(LOGK/2)), exact
    const float hs = (LOGK & 1) ? __fmul_rn(0.70710678118654752f, p2) : p2;

    // X may come from the previous kernel: before the dependency wait only warm L2
    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            const int64_t t = blockIdx.x + (int64_t)i * gridDim.x;
            if (t < M) src.prefetch(t * K, K);
        }
    }
    pdl_launch_dependents();
    pdl_wait_prerequisites();

    for (int64_t t = blockIdx.x; t < M; t += gridDim.x) {
        // the next token's row: one token ahead keeps the rows in flight (two per CTA) well
        // inside L2; two ahead overran it at K = 16384 and rows were read from HBM twice
        if (tid == 0 && t + gridDim.x < M) src.prefetch((t + gridDim.x) * K, K);
        zero_fill(zf, t);  // a following split-K GEMM's output row (and, for token 0, its counters)
        const int64_t row = t * K;

        // phase 0: elements tid + (r << TLOG), pairs (2j, 2j+1)
        float2 v[NP];
#pragma unroll
        for (int j = 0; j < NP; ++j) {
            v[j].x = src.get1(row + tid + ((2 * j) << TLOG));
            v[j].y = src.get1(row + tid + ((2 * j + 1) << TLOG));
        }
        float2 sacc[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) sacc[a] = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int j = 0; j < NP; ++j) sacc[j & 3] = __ffma2_rn(v[j], v[j], sacc[j & 3]);
        const float2 s01 = __fadd2_rn(sacc[0], sacc[1]), s23 = __fadd2_rn(sacc[2], sacc[3]);
        float ss = __fadd_rn(__fadd_rn(s01.x, s01.y), __fadd_rn(s23.x, s23.y));
        asm volatile("" : "+f"(ss));  // keep the sum here, not sunk to its use after phase 1
        if (gain != nullptr) {
#pragma unroll
            for (int j = 0; j < NP; ++j) {
                v[j].x = __fmul_rn(v[j].x, __ldg(gain + tid + ((2 * j) << TLOG)));
                v[j].y = __fmul_rn(v[j].y, __ldg(gain + tid + ((2 * j + 1) << TLOG)));
            }
        }
#pragma unroll
        for (int b = 0; b < ELOG; ++b) butterfly_pairs(v, b);

        // transpose: word stores in the phase-0 layout, 16-byte loads in the phase-1 layout
#pragma unroll
        for (int j = 0; j < NP; ++j) {
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int r = 2 * j + k;
                // bits ELOG..ELOG+2 of element tid + (r << TLOG) are bits of r (TLOG >= 5)
                const int sw = ((r << TLOG) >> ELOG) & 7;
                buf[(tid ^ (sw << 2)) + (r << TLOG)] = k ? v[j].y : v[j].x;
            }
        }
        __syncthreads();
        const float *rb = buf + tid * E;
#pragma unroll
        for (int u = 0; u < E / 4; ++u) {
            const float4 q = *reinterpret_cast<const float4 *>(rb + 4 * ((u & ~7) | ((u ^ tid) & 7)));
            v[2 * u] = make_float2(q.x, q.y);
            v[2 * u + 1] = make_float2(q.z, q.w);
        }
#pragma unroll
        for (int b = 0; b < TLOG; ++b) butterfly_pairs(v, b);

        // one reduction of (sum x^2, max|z| or sum|z|); every thread finishes it
        float st;
        {
            float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};  // four short chains
            if (mean) {
#pragma unroll
                for (int j = 0; j < NP; ++j) {
                    acc[2 * (j & 1)] += fabsf(v[j].x);
                    acc[2 * (j & 1) + 1] += fabsf(v[j].y);
                }
                st = (acc[0] + acc[1]) + (acc[2] + acc[3]);
            } else {
#pragma unroll
                for (int j = 0; j < NP; ++j) {
                    acc[2 * (j & 1)] = fmaxf(acc[2 * (j & 1)], fabsf(v[j].x));
                    acc[2 * (j & 1) + 1] = fmaxf(acc[2 * (j & 1) + 1], fabsf(v[j].y));
                }
                st = fmaxf(fmaxf(acc[0], acc[1]), fmaxf(acc[2], acc[3]));
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            ss += __shfl_xor_sync(0xffffffffu, ss, o);
            const float x = __shfl_xor_sync(0xffffffffu, st, o);
            st = mean ? st + x : fmaxf(st, x);
        }
        if constexpr (W > 1) {
            // red was last read before this token's transpose barrier
            if (lane == 0) red[warp] = make_float2(ss, st);
            __syncthreads();
            float2 q = red[0];
#pragma unroll
            for (int w = 1; w < W; ++w) {
                const float2 p = red[w];
                q.x += p.x;
                q.y = mean ? q.y + p.y : fmaxf(q.y, p.y);
            }
            ss = q.x;
            st = q.y;
        }
        const float rho = __fmul_rn(rms_factor(ss, K, eps), hs);
        const float rs = __fmul_rn(rho, st);
        const float stat = mean ? __fdiv_rn(rs, (float)K) : rs;
        const float s_eff = __fmul_rn(rho, quant_params(stat, eps, mode).s);
        if (tid == 0) scale_x[t] = stat;

        // codes: rne(z * s_eff) by one fused multiply-add with the rounding bias (see
        // quant_bits); int4 clips the biased value, int8 never needs to
        int8_t *out = codes + row + tid * E;
        const float2 s2 = make_float2(s_eff, s_eff), b2 = make_float2(kBias, kBias);
#pragma unroll
        for (int u = 0; u < E / 16; ++u) {
            uint32_t w[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float2 a = __ffma2_rn(v[8 * u + 2 * k], s2, b2);
                float2 c = __ffma2_rn(v[8 * u + 2 * k + 1], s2, b2);
                if (mean) {
                    a.x = fminf(fmaxf(a.x, qlo), qhi);
                    a.y = fminf(fmaxf(a.y, qlo), qhi);
                    c.x = fminf(fmaxf(c.x, qlo), qhi);
                    c.y = fminf(fmaxf(c.y, qlo), qhi);
                }
                w[k] = pack4_perm(__float_as_uint(a.x), __float_as_uint(a.y), __float_as_uint(c.x),
                                  __float_as_uint(c.y));
            }
            *reinterpret_cast<uint4 *>(out + 16 * u) = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
}

// ------------------------------------------------------------------ plain kernel (no FWHT)
// Per-token scalars of the plain kernel, computed once by warp 0 and shared.
struct TokenScalars {
    float rn, stat, s, lo, hi;
};

// Block reduction of (sum, max-or-sum) over a CTA of any whole number of warps.  Every
// warp reduces its own values with shuffles; warp 0 combines the per-warp results and
// runs finish(r) on its lane 0, which writes the token's scalars to *out; the CTA then
// synchronises, so every thread may read *out.
template <class F>
__device__ __forceinline__ void block_reduce2(float ss, float st, bool mean, float2 *red, F finish) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        ss += __shfl_xor_sync(0xffffffffu, ss, o);
        const float t = __shfl_xor_sync(0xffffffffu, st, o);
        st = mean ? st + t : fmaxf(st, t);
    }
    const int W = blockDim.x >> 5;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __syncthreads();  // red and the scalars may still be read from a previous reduction
    if (lane == 0) red[warp] = make_float2(ss, st);
    __syncthreads();
    if (warp == 0) {
        float2 r = lane < W ? red[lane] : make_float2(0.0f, 0.0f);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            r.x += __shfl_xor_sync(0xffffffffu, r.x, o);
            const float t = __shfl_xor_sync(0xffffffffu, r.y, o);
            r.y = mean ? r.y + t : fmaxf(r.y, t);
        }
        if (lane == 0) finish(r);
    }
    __syncthreads();
}

// One CTA of T threads (a multiple of 32, chosen per K and M) per token; thread tid
// owns the 8-element chunks c = it*T + tid, it in [0, NV8); K % 8 == 0.  Without a
// gain the statistics of y = x * r come from those of x in the same pass as sum(x^2):
//   int8:  max_k |fl(x_k r)| = fl(r max_k |x_k|)   (rounding is monotone), exact;
//   int4:  sum_k |fl(x_k r)| = fl(r sum_k |x_k|) up to one rounding per term,
// so one block reduction serves both.  With a gain, y is formed first and reduced
// again.  The scalar steps (IEEE divisions and square root) run once per token, in one
// thread.  Per element the kernel then spends two multiplies, one add and a byte
// permute on the code.
template <int NV8, class Src>
__global__ void __launch_bounds__(512)
act_quant_plain_kernel(Src src, const float *__restrict__ gain, int K, float eps,
                       int mode, int8_t *__restrict__ codes, float *__restrict__ scale_x, ZeroFill zf) {
    __shared__ float2 red[32];
    __shared__ TokenScalars ts;
    pdl_launch_dependents();  // as in the FWHT kernel: the GEMM may launch, X is waited for
    if (threadIdx.x == 0) src.prefetch((int64_t)blockIdx.x * K, K);  // warm L2 while the producer finishes
    pdl_wait_prerequisites();
    zero_fill(zf, blockIdx.x);
    const int tid = threadIdx.x, T = blockDim.x;
    const int64_t row = (int64_t)blockIdx.x * K;
    const int K8 = K >> 3;
    const bool mean = mode != BITNET_ACT_INT8_ABSMAX;
    const bool nogain = gain == nullptr;
    float v[NV8][8];
#pragma unroll
    for (int it = 0; it < NV8; ++it) {
        const int c = it * T + tid;
        if (c < K8) {
            src.get8(row + 8 * c, v[it]);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) v[it][e] = 0.0f;
        }
    }
    float ss = 0.0f, st = 0.0f;
    if (mean) {
#pragma unroll
        for (int it = 0; it < NV8; ++it)
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                ss = fmaf(v[it][e], v[it][e], ss);
                st += fabsf(v[it][e]);
            }
    } else {
#pragma unroll
        for (int it = 0; it < NV8; ++it)
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                ss = fmaf(v[it][e], v[it][e], ss);
                st = fmaxf(st, fabsf(v[it][e]));
            }
    }
    block_reduce2(ss, st, mean, red, [&](float2 r) {
        ts.rn = rms_factor(r.x, K, eps);
        if (nogain) {
            const float ry = __fmul_rn(ts.rn, r.y);
            ts.stat = mean ? __fdiv_rn(ry, (float)K) : ry;
            const QuantParams q = quant_params(ts.stat, eps, mode);
            ts.s = q.s;
            ts.lo = q.lo;
            ts.hi = q.hi;
        }
    });
    const float rn = ts.rn;
    if (nogain) {
#pragma unroll
        for (int it = 0; it < NV8; ++it)
#pragma unroll
            for (int e = 0; e < 8; ++e) v[it][e] = __fmul_rn(v[it][e], rn);
    } else {
        float part = 0.0f;
#pragma unroll
        for (int it = 0; it < NV8; ++it) {
            const int c = it * T + tid;
            float g[8];
            if (c < K8) {
                const float4 g0 = __ldg(reinterpret_cast<const float4 *>(gain) + 2 * c);
                const float4 g1 = __ldg(reinterpret_cast<const float4 *>(gain) + 2 * c + 1);
                g[0] = g0.x; g[1] = g0.y; g[2] = g0.z; g[3] = g0.w;
                g[4] = g1.x; g[5] = g1.y; g[6] = g1.z; g[7] = g1.w;
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) g[e] = 0.0f;
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float y = __fmul_rn(__fmul_rn(v[it][e], rn), g[e]);
                v[it][e] = y;
                part = mean ? part + fabsf(y) : fmaxf(part, fabsf(y));
            }
        }
        block_reduce2(0.0f, part, mean, red, [&](float2 r) {
            ts.stat = mean ? __fdiv_rn(r.y, (float)K) : r.y;
            const QuantParams q = quant_params(ts.stat, eps, mode);
            ts.s = q.s;
            ts.lo = q.lo;
            ts.hi = q.hi;
        });
    }
    const float qs = ts.s, qlo = ts.lo, qhi = ts.hi;
    // int8: |y| <= gamma makes |y*s| < 127.5, so the clip can never act.
#pragma unroll
    for (int it = 0; it < NV8; ++it) {
        const int c = it * T + tid;
        if (c < K8) {
            uint32_t f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = quant_bits(v[it][e], qs, qlo, qhi, mean);
            *reinterpret_cast<uint2 *>(codes + row + 8 * c) =
                make_uint2(pack4_perm(f[0], f[1], f[2], f[3]), pack4_perm(f[4], f[5], f[6], f[7]));
        }
    }
    if (tid == 0) scale_x[blockIdx.x] = ts.stat;
}

// Launch with programmatic stream serialisation: the kernel may start while the
// previous kernel of the stream finishes.  It lets its own dependents launch at once
// and waits (griddepcontrol.wait) before reading anything; the dependents in turn
// only prefetch weights into L2 before their own wait.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

template <int LOGK, class Src>
cudaError_t launch_fwht(const Src &src, int64_t M, const float *gain, float eps, int mode, int8_t *codes,
                        float *scale_x, const ZeroFill &zf, cudaStream_t s) {
    using S = FwhtShape<LOGK>;
    const size_t smem = (size_t)(S::K + S::K / 32) * sizeof(float);
    auto kern = act_quant_fwht_kernel<LOGK, Src>;
    if (smem > 48 * 1024) {
        static bool done[kMaxDevices] = {};
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev >= kMaxDevices || !done[dev]) {
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
            if (dev < kMaxDevices) done[dev] = true;
        }
    }
    return launch_pdl(kern, dim3((unsigned)M), dim3(S::T), smem, s, src, gain, eps, mode, codes, scale_x, zf);
}

// The streaming kernel for K = 2^LOGK, 11 <= LOGK <= 14: a persistent grid of as many
// CTAs as the SMs hold.
template <int LOGK, class Src>
cudaError_t launch_fwht_stream(const Src &src, int64_t M, const float *gain, float eps, int mode, int8_t *codes,
                               float *scale_x, const ZeroFill &zf, cudaStream_t s) {
    using S = StreamShape<LOGK>;
    auto kern = act_quant_fwht_stream_kernel<LOGK, Src>;
    static int bps[kMaxDevices] = {};  // resident CTAs per SM
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int per_sm = dev < kMaxDevices ? bps[dev] : 0;
    if (per_sm == 0) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM);
        if (e != cudaSuccess) return e;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, S::T, S::SMEM);
        if (e != cudaSuccess || per_sm < 1) per_sm = 1;
        if (dev < kMaxDevices) bps[dev] = per_sm;
    }
    const int64_t slots = (int64_t)per_sm * sm_count();
    const int grid = (int)(M < slots ? M : slots);
    return launch_pdl(kern, dim3((unsigned)grid), dim3(S::T), (size_t)S::SMEM, s, src, gain, eps, mode, M, codes,
                      scale_x, zf);
}

template <int NV8, class Src>
cudaError_t launch_plain(const Src &src, int64_t M, int K, int T, const float *gain, float eps, int mode,
                         int8_t *codes, float *scale_x, const ZeroFill &zf, cudaStream_t s) {
    return launch_pdl(act_quant_plain_kernel<NV8, Src>, dim3((unsigned)M), dim3(T), 0, s, src, gain, K, eps, mode,
                      codes, scale_x, zf);
}

// Many tokens of a plain input with 2^11 <= K <= 2^14: the streaming FWHT kernel.  The
// SwiGLU source stays on the per-token kernel: inlined 128 times per thread, its exp and
// IEEE division made the streaming kernel several times slower (0.11 of HBM on the
// 2048 x 8192 Wdown input against 0.4 per token).
template <class Src>
cudaError_t dispatch_stream(const Src &, int64_t, int, const float *, float, int, int8_t *, float *, const ZeroFill &,
                            cudaStream_t, bool &used) {
    used = false;
    return cudaSuccess;
}
template <bool BF16>
cudaError_t dispatch_stream(const XSrc<BF16> &src, int64_t M, int K, const float *gain, float eps, int mode,
                            int8_t *codes, float *scale_x, const ZeroFill &zf, cudaStream_t s, bool &used) {
    used = M >= 2 * (int64_t)sm_count();
    if (!used) return cudaSuccess;
    switch (__builtin_ctz((unsigned)K)) {
        case 11: return launch_fwht_stream<11>(src, M, gain, eps, mode, codes, scale_x, zf, s);
        case 12: return launch_fwht_stream<12>(src, M, gain, eps, mode, codes, scale_x, zf, s);
        case 13: return launch_fwht_stream<13>(src, M, gain, eps, mode, codes, scale_x, zf, s);
        case 14: return launch_fwht_stream<14>(src, M, gain, eps, mode, codes, scale_x, zf, s);
        default: used = false; return cudaSuccess;
    }
}

template <class Src>
cudaError_t dispatch(const Src &src, int64_t M, int K, const float *gain, float eps, int fwht, int mode,
                     int8_t *codes, float *scale_x, const ZeroFill &zf, cudaStream_t s) {
    if (fwht) {
        bool used = false;
        const cudaError_t e = dispatch_stream(src, M, K, gain, eps, mode, codes, scale_x, zf, s, used);
        if (used) return e;
        switch (__builtin_ctz((unsigned)K)) {
            case 7: return launch_fwht<7>(src, M, gain, eps, mode, codes, scale_x, zf, s);
            case 8: return launch_fwht<8>(src, M, gain, eps, mode, codes, scale_x, zf, s);
            case 9: return launch_fwht<9>(src, M, gain, eps, mode, codes, scale_x, zf, s);
            case 10: return launch_fwht<10>(src, M, gain, eps, mode, codes, scale_x, zf, s);
            case 11: return launch_fwht<11>(src, M, gain, eps, mode, codes, scale_x, zf, s);
            case 12: return launch_fwht<12>(src, M, gain, eps, mode, codes, scale_x, zf, s);
            case 13: return launch_fwht<13>(src, M, gain, eps, mode, codes, scale_x, zf, s);
            case 14: return launch_fwht<14>(src, M, gain, eps, mode, codes, scale_x, zf, s);
            case 15: return launch_fwht<15>(src, M, gain, eps, mode, codes, scale_x, zf, s);
            default: return cudaErrorInvalidValue;
        }
    }
    // Few tokens (decode): about 256 threads per token, so each thread's serial work
    // stays short.  Many tokens: 32 elements per thread (8 for short rows, 64 for
    // K > 16384), so each CTA's per-token work is spread over more elements.  At most
    // 512 threads.
    const int k8 = K / 8;
    int nv8;
    if (M <= 64) nv8 = k8 <= 256 ? 1 : (k8 <= 512 ? 2 : (k8 <= 1024 ? 4 : 8));
    else nv8 = k8 < 128 ? 1 : (k8 <= 2048 ? 4 : 8);
    const int T = (int)ceil_div(ceil_div(k8, nv8), 32) * 32;
    if (T > 512) return cudaErrorInvalidValue;
    if (nv8 == 1) return launch_plain<1>(src, M, K, T, gain, eps, mode, codes, scale_x, zf, s);
    if (nv8 == 2) return launch_plain<2>(src, M, K, T, gain, eps, mode, codes, scale_x, zf, s);
    if (nv8 == 4) return launch_plain<4>(src, M, K, T, gain, eps, mode, codes, scale_x, zf, s);
    return launch_plain<8>(src, M, K, T, gain, eps, mode, codes, scale_x, zf, s);
}

}  // namespace

// Host entries used by the ABI layer (arguments already validated).
cudaError_t launch_act_quant(const void *X, bool bf16, int64_t M, int K, const float *gain, float eps,
                             int fwht, int mode, int8_t *codes, float *scale_x, cudaStream_t s, ZeroFill zf) {
    if (M == 0) return cudaSuccess;
    return bf16 ? dispatch(XSrc<true>{X}, M, K, gain, eps, fwht, mode, codes, scale_x, zf, s)
                : dispatch(XSrc<false>{X}, M, K, gain, eps, fwht, mode, codes, scale_x, zf, s);
}

cudaError_t launch_act_quant_swiglu(const void *gate, const void *up, bool bf16, int64_t M, int K, const float *gain,
                                    float eps, int fwht, int mode, int8_t *codes, float *scale_x, cudaStream_t s,
                                    ZeroFill zf) {
    if (M == 0) return cudaSuccess;
    return bf16 ? dispatch(SwigluSrc<true>{gate, up}, M, K, gain, eps, fwht, mode, codes, scale_x, zf, s)
                : dispatch(SwigluSrc<false>{gate, up}, M, K, gain, eps, fwht, mode, codes, scale_x, zf, s);
}

}  // namespace bitnet
