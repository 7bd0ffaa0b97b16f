// landmarks.cu -- DHSA chunk landmarks l = sqrt(S) * mean of the chunk's keys
// (Dynamic Hierarchical Sparse Attention review, "What carries the argument").
//
// HBM-bound: every key is read once (16-byte streaming loads, fully coalesced:
// one chunk is S*d contiguous elements) and one fp32 row per chunk is written.
// A 256-thread block reduces one chunk at a time: each thread owns one 16-byte
// column slice and S/rows_per_pass rows of it, then the per-slice partial sums
// are folded through shared memory.
#include "common.cuh"

namespace hsa {

template <typename T, int D, int S>
__global__ void __launch_bounds__(256)
landmarks_kernel(const T *__restrict__ K, float *__restrict__ lm, int64_t n_chunks_total,
                 int64_t L, int64_t Nc, float inv_sqrt_s_times_s) {
    constexpr int VEC = Vec16<T>::N;          // elements per 16-byte load
    constexpr int LPR = D / VEC;              // threads per key row
    constexpr int RPP = 256 / LPR;            // rows per pass
    constexpr int PASSES = S / RPP;
    static_assert(S % RPP == 0, "chunk must be a whole number of passes");
    __shared__ float part[RPP][D + 4];

    const int tid = threadIdx.x;
    const int col = (tid % LPR) * VEC;
    const int row = tid / LPR;
    for (int64_t ci = blockIdx.x; ci < n_chunks_total; ci += gridDim.x) {
        const int64_t bg = ci / Nc, i = ci % Nc;
        const T *src = K + (bg * L + i * S) * D;
        float acc[VEC];
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
        uint4 raw[PASSES];
#pragma unroll
        for (int p = 0; p < PASSES; ++p)
            raw[p] = ld_stream16(src + (int64_t)(p * RPP + row) * D + col);
#pragma unroll
        for (int p = 0; p < PASSES; ++p) {
            float f[VEC];
            Vec16<T>::unpack(raw[p], f);
#pragma unroll
            for (int e = 0; e < VEC; ++e) acc[e] += f[e];
        }
#pragma unroll
        for (int e = 0; e < VEC; ++e) part[row][col + e] = acc[e];
        __syncthreads();
        if (tid < D) {
            float s = 0.f;
#pragma unroll 8
            for (int r = 0; r < RPP; ++r) s += part[r][tid];
            // sqrt(S) * (sum / S); for S = 64 this is sum * 0.125 exactly.
            lm[ci * D + tid] = s * inv_sqrt_s_times_s;
        }
        __syncthreads();
    }
}

template <typename T, int D>
static cudaError_t launch_landmarks_t(const void *K, float *lm, int B, int Hkv, int64_t L,
                                      cudaStream_t st) {
    constexpr int S = 64;
    const int64_t Nc = L / S;
    const int64_t total = (int64_t)B * Hkv * Nc;
    if (total == 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t grid = total < (int64_t)sms * 8 ? total : (int64_t)sms * 8;
    const float f = 1.0f / sqrtf((float)S);   // sqrt(S)/S
    landmarks_kernel<T, D, S><<<(unsigned)grid, 256, 0, st>>>((const T *)K, lm, total, L, Nc, f);
    return cudaGetLastError();
}

cudaError_t launch_landmarks(const void *K, bool bf16, float *lm, int B, int Hkv, int64_t L,
                             int d, cudaStream_t st) {
    if (bf16) {
        return d == 128 ? launch_landmarks_t<__nv_bfloat16, 128>(K, lm, B, Hkv, L, st)
                        : launch_landmarks_t<__nv_bfloat16, 64>(K, lm, B, Hkv, L, st);
    }
    return d == 128 ? launch_landmarks_t<float, 128>(K, lm, B, Hkv, L, st)
                    : launch_landmarks_t<float, 64>(K, lm, B, Hkv, L, st);
}

}  // namespace hsa
