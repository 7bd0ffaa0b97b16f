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

// ---------------------------------------------------------------- incremental update
// Landmarks of the chunks that completed while a cache grew from len0[b] to
// len1[b] tokens: chunks len0[b]/S .. len1[b]/S - 1 of sequence b (lengths
// clamped to 0 .. Lmax).  One warp per chunk, lanes over 16-byte column
// slices, 32 / (D / VEC) rows per step; partial rows folded by shuffles.
template <typename T, typename TL, int D>
__global__ void __launch_bounds__(256)
landmarks_append_kernel(const T *__restrict__ K, TL *__restrict__ lm, int Hkv, int64_t Lmax,
                        int S, const int32_t *__restrict__ len0, const int32_t *__restrict__ len1) {
    constexpr int VEC = Vec16<T>::N;
    constexpr int LPR = D / VEC;                              // lanes per row slice
    constexpr int RPS = 32 / LPR;                             // rows per warp step
    const int64_t bg = blockIdx.x;
    const int64_t b = bg / Hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t Nmax = Lmax / S;
    auto clampl = [&](int64_t v) { return v < 0 ? (int64_t)0 : v > Lmax ? Lmax : v; };
    const int64_t lo = clampl(len0[b]) / S, hi = clampl(len1[b]) / S;
    const int col = (lane % LPR) * VEC, r0 = lane / LPR;
    const float f = rsqrtf((float)S);                         // sqrt(S) * (sum / S)
    for (int64_t c = lo + (int64_t)blockIdx.y * 8 + warp; c < hi; c += (int64_t)gridDim.y * 8) {
        const T *src = K + (bg * Lmax + c * S) * D + col;
        float acc[VEC];
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
        for (int r = r0; r < S; r += RPS) {
            float v[VEC];
            Vec16<T>::unpack(ld_stream16(src + (int64_t)r * D), v);
#pragma unroll
            for (int e = 0; e < VEC; ++e) acc[e] += v[e];
        }
#pragma unroll
        for (int o = LPR; o < 32; o <<= 1)
#pragma unroll
            for (int e = 0; e < VEC; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
        if (lane < LPR) {
            TL *dst = lm + (bg * Nmax + c) * D + col;
#pragma unroll
            for (int e = 0; e < VEC; ++e) dst[e] = from_f32<TL>(acc[e] * f);
        }
    }
}

cudaError_t launch_landmarks_append(const void *K, bool bf16, void *lm, bool lm_bf16, int B,
                                    int Hkv, int64_t Lmax, int d, int S, const int32_t *len0,
                                    const int32_t *len1, int max_new_chunks, cudaStream_t st) {
    const int64_t pairs = (int64_t)B * Hkv;
    if (pairs == 0 || Lmax / S == 0) return cudaSuccess;
    int ny = (max_new_chunks + 7) / 8;
    if (ny < 1) ny = 1;
    if (ny > 1024) ny = 1024;
    const dim3 grid((unsigned)pairs, (unsigned)ny);
    using bf = __nv_bfloat16;
#define HSA_APPEND(T, TL, DD) \
    landmarks_append_kernel<T, TL, DD><<<grid, 256, 0, st>>>((const T *)K, (TL *)lm, Hkv, Lmax, S, len0, len1)
    if (bf16) {
        if (lm_bf16) { if (d == 128) HSA_APPEND(bf, bf, 128); else HSA_APPEND(bf, bf, 64); }
        else { if (d == 128) HSA_APPEND(bf, float, 128); else HSA_APPEND(bf, float, 64); }
    } else {
        if (lm_bf16) { if (d == 128) HSA_APPEND(float, bf, 128); else HSA_APPEND(float, bf, 64); }
        else { if (d == 128) HSA_APPEND(float, float, 128); else HSA_APPEND(float, float, 64); }
    }
#undef HSA_APPEND
    return cudaGetLastError();
}

// ---------------------------------------------------------------- variable-length chunks
// Checks the boundaries (0 = b_0 < b_1 < ... < b_n = L, no chunk longer than
// 64 tokens) in one block and stores the verdict in bs[n + 1].  Wrong
// boundaries also set kFlagBadBounds in the status word (hsa_check reports
// them).
__global__ void __launch_bounds__(1024)
varlen_check_kernel(const int32_t *__restrict__ bounds, int64_t n, int64_t L,
                    int32_t *__restrict__ bs, unsigned *__restrict__ status) {
    bool bad = false;
    for (int64_t c = threadIdx.x; c < n; c += blockDim.x) {
        const int64_t lo = bounds[c], hi = bounds[c + 1];
        bad |= hi <= lo || hi - lo > kMaxVarChunk || lo < 0 || hi > L;
        bad |= c == 0 && lo != 0;
        bad |= c == n - 1 && hi != L;
    }
    bad = __syncthreads_or(bad);
    if (threadIdx.x == 0) {
        bs[n + 1] = bad ? 1 : 0;
        if (bad) atomicOr(status, kFlagBadBounds);
    }
}

// The boundaries every later kernel reads, bs[0..n], and tok_chunk[t] = the
// chunk holding token t.  bs is a copy of the caller's boundaries when they
// passed the check and an even split of the L tokens into n chunks otherwise
// (each 1..64 tokens, as n <= L <= 64 n), so that no kernel of a call with
// wrong boundaries reads or writes outside its buffers.  One thread per chunk.
__global__ void __launch_bounds__(256)
varlen_setup_kernel(const int32_t *__restrict__ bounds, int64_t n, int64_t L,
                    int32_t *__restrict__ bs, int32_t *__restrict__ tok_chunk) {
    const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= n) return;
    const bool bad = bs[n + 1] != 0;
    const int64_t lo = bad ? c * L / n : bounds[c];
    const int64_t hi = bad ? (c + 1) * L / n : bounds[c + 1];
    bs[c] = (int32_t)lo;
    if (c == n - 1) bs[n] = (int32_t)hi;
    for (int64_t t = lo; t < hi; ++t) tok_chunk[t] = (int32_t)c;
}

// sqrt(|C|) * mean of the keys of each variable-length chunk = sum / sqrt(|C|):
// one warp per (b, g, chunk), lanes over 16-byte column slices.
template <typename T, int D>
__global__ void __launch_bounds__(256)
landmarks_varlen_kernel(const T *__restrict__ K, float *__restrict__ lm, int64_t total,
                        Chunks ch, int64_t n) {
    constexpr int VEC = Vec16<T>::N;
    constexpr int LPR = D / VEC;                              // lanes per row slice
    const int lane = threadIdx.x & 31;
    const int64_t w = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (w >= total) return;
    const int64_t bg = w / n, i = w % n;
    const int64_t first = chunk_first(ch, i);
    const int len = chunk_len(ch, i);
    const int rows_per_step = 32 / LPR;                       // rows a warp reads at once
    const int col = (lane % LPR) * VEC, r0 = lane / LPR;
    float acc[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
    for (int r = r0; r < len; r += rows_per_step) {
        if (first + r >= ch.L) break;
        float f[VEC];
        Vec16<T>::unpack(ld_stream16(K + (bg * ch.L + first + r) * D + col), f);
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[e] += f[e];
    }
    // fold the rows_per_step partial rows (lanes with equal column slices)
#pragma unroll
    for (int o = LPR; o < 32; o <<= 1)
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
    if (lane < LPR) {
        const float f = len > 0 ? rsqrtf((float)len) : 0.f;
        float *dst = lm + w * D + col;
#pragma unroll
        for (int e = 0; e < VEC; ++e) dst[e] = acc[e] * f;
    }
}

cudaError_t launch_varlen_setup(const int32_t *bounds, int64_t n, int64_t L, int32_t *bs,
                                int32_t *tok_chunk, unsigned *status, cudaStream_t st) {
    varlen_check_kernel<<<1, 1024, 0, st>>>(bounds, n, L, bs, status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    varlen_setup_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(bounds, n, L, bs, tok_chunk);
    return cudaGetLastError();
}

cudaError_t launch_landmarks_varlen(const void *K, bool bf16, float *lm, int B, int Hkv, int64_t L,
                                    int d, const int32_t *bounds, int64_t n, cudaStream_t st) {
    const int64_t total = (int64_t)B * Hkv * n;
    if (total == 0) return cudaSuccess;
    Chunks ch = {bounds, nullptr, L, 64};
    const unsigned grid = (unsigned)((total + 7) / 8);
    if (bf16) {
        if (d == 128) landmarks_varlen_kernel<__nv_bfloat16, 128><<<grid, 256, 0, st>>>((const __nv_bfloat16 *)K, lm, total, ch, n);
        else landmarks_varlen_kernel<__nv_bfloat16, 64><<<grid, 256, 0, st>>>((const __nv_bfloat16 *)K, lm, total, ch, n);
    } else {
        if (d == 128) landmarks_varlen_kernel<float, 128><<<grid, 256, 0, st>>>((const float *)K, lm, total, ch, n);
        else landmarks_varlen_kernel<float, 64><<<grid, 256, 0, st>>>((const float *)K, lm, total, ch, n);
    }
    return cudaGetLastError();
}

}  // namespace hsa
