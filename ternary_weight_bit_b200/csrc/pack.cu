// pack.cu -- step 4a: absmean ternarisation of a weight matrix and 2-bit packing.
//
// Method: bitnet_v2_engine.py page, Eq. 1/2 and quantize_weight_ternary
// (alpha = mean|W| per tensor, t = RoundClip(W / (alpha + eps), -1, 1)); the code map
// t -> t + 1 of the tl2_lookup_simulation listing (youngju.dev BitNet transcription);
// pack once / forward many as in bitnet_cpp_edge.py's prepare_weights.
//
// Three kernels, all deterministic for a given (N, K):
//   1. abs_sum_partial: a fixed grid of kSumBlocks blocks each sums |W| over a
//      contiguous slice in double, reducing in a fixed tree order;
//   2. alpha_finalize: one block sums the partials in a fixed order and rounds
//      sum / (N*K) once to float;
//   3. pack_words: one thread per 32-bit packed word (16 weights): IEEE division
//      W / (alpha + eps), round half to even, clip to [-1, 1], place code t + 1 at
//      bits [4i + 2h, 4i + 2h + 2) for k = 16w + 8h + i.
#include "common.cuh"

namespace bitnet {

constexpr int kSumBlocks = 1184;  // 8 x 148 SMs
constexpr int kSumThreads = 256;

namespace {

__device__ __forceinline__ double block_sum_d(double v, double *red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    double s = 0.0;
    if (warp == 0) {
        s = lane < (int)(blockDim.x >> 5) ? red[lane] : 0.0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    }
    return s;  // valid in thread 0
}

__global__ void __launch_bounds__(kSumThreads)
abs_sum_partial(const float *__restrict__ W, int64_t count, double *__restrict__ partial) {
    __shared__ double red[32];
    const int64_t per = ceil_div(ceil_div(count, kSumBlocks), 4) * 4;  // multiple of 4 elements
    const int64_t b0 = (int64_t)blockIdx.x * per;
    const int64_t b1 = b0 + per < count ? b0 + per : count;
    double acc = 0.0;
    // count is a multiple of 4 (K % 128 == 0), so float4 groups never straddle the end.
    for (int64_t i = b0 + 4 * (int64_t)threadIdx.x; i < b1; i += 4 * kSumThreads) {
        const float4 v = __ldg(reinterpret_cast<const float4 *>(W + i));
        acc += fabs((double)v.x) + fabs((double)v.y) + fabs((double)v.z) + fabs((double)v.w);
    }
    acc = block_sum_d(acc, red);
    if (threadIdx.x == 0) partial[blockIdx.x] = acc;
}

__global__ void __launch_bounds__(1024)
alpha_finalize(const double *__restrict__ partial, int64_t count, float *__restrict__ alpha) {
    __shared__ double red[32];
    double acc = 0.0;
    for (int i = threadIdx.x; i < kSumBlocks; i += blockDim.x) acc += partial[i];
    acc = block_sum_d(acc, red);
    if (threadIdx.x == 0) *alpha = (float)(acc / (double)count);
}

__global__ void __launch_bounds__(256)
pack_words(const float *__restrict__ W, int64_t words, float eps, const float *__restrict__ alpha,
           uint32_t *__restrict__ packed) {
    const int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (w >= words) return;
    const float d = __fadd_rn(*alpha, eps);
    const float4 *src = reinterpret_cast<const float4 *>(W + 16 * w);  // row-major: word w covers 16 k
    float v[16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float4 f = __ldg(src + q);
        v[4 * q] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
    }
    uint32_t out = 0;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        const float t = fminf(fmaxf(rintf(__fdiv_rn(v[k], d)), -1.0f), 1.0f);
        const uint32_t code = (uint32_t)((int)t + 1);
        const int h = k >> 3, i = k & 7;
        out |= code << (4 * i + 2 * h);
    }
    packed[w] = out;
    // The GEMV/GEMM kernels of a following forward may load packed weights before their
    // programmatic-launch dependency wait (they can launch as soon as this grid exits).
    // The fence makes this thread's store visible device-wide before the grid exits.
    __threadfence();
}

}  // namespace

size_t pack_workspace_bytes() { return (size_t)kSumBlocks * sizeof(double); }

cudaError_t launch_pack(const float *W, int64_t N, int64_t K, float eps, uint8_t *packed, float *alpha,
                        void *ws, cudaStream_t s) {
    const int64_t count = N * K;
    double *partial = reinterpret_cast<double *>(ws);
    abs_sum_partial<<<kSumBlocks, kSumThreads, 0, s>>>(W, count, partial);
    alpha_finalize<<<1, 1024, 0, s>>>(partial, count, alpha);
    const int64_t words = count / 16;
    pack_words<<<(unsigned)ceil_div(words, 256), 256, 0, s>>>(W, words, eps, alpha,
                                                              reinterpret_cast<uint32_t *>(packed));
    return cudaGetLastError();
}

}  // namespace bitnet
