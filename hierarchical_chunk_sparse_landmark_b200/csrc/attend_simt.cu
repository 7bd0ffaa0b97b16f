// attend_simt.cu -- in-chunk attention + score-weighted fusion on CUDA cores.
//
// O[t,h] = sum_k w[t,h,k] * softmax_j(scale q.k_j) V over chunk sel_k
//          + (own_chunk ? causal softmax attention over keys c_t*S .. t : 0)
// (HiLS Attention abstract: attention inside each retrieved chunk, outputs
// fused by retrieval scores.)
//
// Query-centric: one block per (b, t, g), one warp per query head of the
// group.  For every selected chunk the block stages the chunk's K and V rows
// in shared memory; each warp computes its head's 64 logits (lane j: keys j
// and j+32), the chunk softmax with warp shuffles, and P.V with lanes over
// the head dimension, accumulating w_k * o_k in registers.  This is the fp32
// path (fp32 accumulate end to end) and the reference layout for the
// tensor-core path.
//
// Union-softmax variant (one softmax over the keys of all selected chunks and
// the own chunk; Dynamic Hierarchical Sparse Attention review): the chunk
// results are folded with a running maximum instead of the fusion weights,
// acc = sum_k e^{m_k - M} P_k V_k, den = sum_k e^{m_k - M} sum P_k, O = acc / den.
#include "common.cuh"

namespace hsa {

template <typename T, int D>
__global__ void attend_simt_kernel(const T *__restrict__ Q, const T *__restrict__ K,
                                   const T *__restrict__ V, const int32_t *__restrict__ idx,
                                   const float *__restrict__ w, int H, int Hkv, int64_t L, int S,
                                   int topk, int own_chunk, float scale, int union_softmax,
                                   Chunks ch, T *__restrict__ O) {
    constexpr int VEC = Vec16<T>::N;
    constexpr int PAD = VEC;                     // 16 bytes of padding per row
    constexpr int RS = D + PAD;                  // row stride (elements)
    constexpr int MAXS = 64;
    extern __shared__ float4 smem4[];
    float *qs = reinterpret_cast<float *>(smem4);                 // [G][D]
    const int G = H / Hkv;
    T *ks = reinterpret_cast<T *>(qs + G * D);                    // [S][RS]
    T *vs = ks + MAXS * RS;                                       // [S][RS]

    const int64_t t = blockIdx.x;
    const int g = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nthr = blockDim.x;
    const int64_t row = (int64_t)b * L + t;

    for (int e = threadIdx.x; e < G * D; e += nthr)
        qs[e] = to_f32(Q[(row * H + (int64_t)g * G) * D + e]);

    constexpr int R = D / 32;                    // output elements per lane
    float acc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r] = 0.f;
    float run_m = -INFINITY, run_den = 0.f;      // union softmax: running max and sum

    const int64_t c_t = chunk_of(ch, t);
    const T *Kbg = K + ((int64_t)b * Hkv + g) * L * D;
    const T *Vbg = V + ((int64_t)b * Hkv + g) * L * D;
    const int32_t *ip = idx + (row * Hkv + g) * topk;
    const int h = g * G + warp;
    const int n_items = topk + (own_chunk ? 1 : 0);
    for (int it = 0; it < n_items; ++it) {
        int64_t first;
        int nkeys;
        float wt;
        if (it < topk) {
            const int32_t ci = ip[it];
            if (ci < 0) continue;                    // uniform across the block
            first = chunk_first(ch, ci);
            nkeys = chunk_len(ch, ci);
            wt = union_softmax ? 1.f : w[(row * H + h) * topk + it];
        } else {
            first = chunk_first(ch, c_t);
            nkeys = (int)(t - first + 1);
            wt = 1.f;
        }
        __syncthreads();
        const int vec_per_row = D / VEC;
        for (int e = threadIdx.x; e < nkeys * vec_per_row; e += nthr) {
            const int r = e / vec_per_row, c = (e % vec_per_row) * VEC;
            const bool in = first + r < L;             // clamped boundaries stay in the cache
            *reinterpret_cast<uint4 *>(ks + r * RS + c) =
                in ? *reinterpret_cast<const uint4 *>(Kbg + (first + r) * D + c) : make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4 *>(vs + r * RS + c) =
                in ? *reinterpret_cast<const uint4 *>(Vbg + (first + r) * D + c) : make_uint4(0, 0, 0, 0);
        }
        __syncthreads();
        // logits for keys lane and lane+32
        const float *qh = qs + warp * D;
        float lg[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int j = lane + 32 * u;
            lg[u] = -INFINITY;
            if (j < nkeys) {
                float a = 0.f;
#pragma unroll 4
                for (int c = 0; c < D; c += VEC) {
                    float f[VEC];
                    Vec16<T>::unpack(*reinterpret_cast<const uint4 *>(ks + j * RS + c), f);
#pragma unroll
                    for (int e = 0; e < VEC; ++e) a = fmaf(qh[c + e], f[e], a);
                }
                lg[u] = scale * a;
            }
        }
        float mx = fmaxf(lg[0], lg[1]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float p[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) p[u] = (lane + 32 * u < nkeys) ? expf(lg[u] - mx) : 0.f;
        float den = p[0] + p[1];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
        float o_r[R];
#pragma unroll
        for (int r = 0; r < R; ++r) o_r[r] = 0.f;
        for (int j = 0; j < nkeys; ++j) {
            const float pj = __shfl_sync(0xffffffffu, p[j >> 5], j & 31);
#pragma unroll
            for (int r = 0; r < R; ++r) o_r[r] = fmaf(pj, to_f32(vs[j * RS + lane + 32 * r]), o_r[r]);
        }
        if (!union_softmax) {
            const float f = wt / den;
#pragma unroll
            for (int r = 0; r < R; ++r) acc[r] = fmaf(f, o_r[r], acc[r]);
        } else {
            const float m_new = fmaxf(run_m, mx);
            const float c_old = run_m > -INFINITY ? expf(run_m - m_new) : 0.f;
            const float c_new = expf(mx - m_new);
            run_den = run_den * c_old + den * c_new;
#pragma unroll
            for (int r = 0; r < R; ++r) acc[r] = acc[r] * c_old + o_r[r] * c_new;
            run_m = m_new;
        }
    }
    if (union_softmax) {
        const float inv = run_den > 0.f ? 1.f / run_den : 0.f;
#pragma unroll
        for (int r = 0; r < R; ++r) acc[r] *= inv;
    }
    T *op = O + (row * H + h) * (int64_t)D;
#pragma unroll
    for (int r = 0; r < R; ++r) op[lane + 32 * r] = from_f32<T>(acc[r]);
}

template <typename T, int D>
static cudaError_t launch_attend_simt_t(const void *Q, const void *K, const void *V,
                                        const int32_t *idx, const float *w, int B, int H,
                                        int Hkv, int64_t L, int S, int topk, int own_chunk,
                                        float scale, int union_softmax, Chunks ch, void *O,
                                        cudaStream_t st) {
    constexpr int VEC = Vec16<T>::N;
    const int G = H / Hkv;
    const size_t smem = sizeof(float) * G * D + 2 * sizeof(T) * 64 * (D + VEC);
    auto kern = attend_simt_kernel<T, D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)L, (unsigned)Hkv, (unsigned)B);
    kern<<<grid, 32 * G, smem, st>>>((const T *)Q, (const T *)K, (const T *)V, idx, w, H, Hkv,
                                     L, S, topk, own_chunk, scale, union_softmax, ch, (T *)O);
    return cudaGetLastError();
}

cudaError_t launch_attend_simt(const void *Q, const void *K, const void *V, bool bf16,
                               const int32_t *idx, const float *w, int B, int H, int Hkv,
                               int64_t L, int d, int S, int topk, int own_chunk, float scale,
                               int union_softmax, const int32_t *bounds, const int32_t *tok_chunk,
                               void *O, cudaStream_t st) {
    const Chunks ch = {bounds, tok_chunk, L, S};
    if (bf16)
        return d == 128 ? launch_attend_simt_t<__nv_bfloat16, 128>(Q, K, V, idx, w, B, H, Hkv, L, S, topk, own_chunk, scale, union_softmax, ch, O, st)
                        : launch_attend_simt_t<__nv_bfloat16, 64>(Q, K, V, idx, w, B, H, Hkv, L, S, topk, own_chunk, scale, union_softmax, ch, O, st);
    return d == 128 ? launch_attend_simt_t<float, 128>(Q, K, V, idx, w, B, H, Hkv, L, S, topk, own_chunk, scale, union_softmax, ch, O, st)
                    : launch_attend_simt_t<float, 64>(Q, K, V, idx, w, B, H, Hkv, L, S, topk, own_chunk, scale, union_softmax, ch, O, st);
}

}  // namespace hsa
