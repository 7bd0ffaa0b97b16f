// decode.cu -- one new query per sequence against a long KV cache.
//
// D1  group score of every chunk:  sbar_i = scale * qbar . l_i, i < Lc/S
// D2  top-K over all chunks (score desc, index asc)
// D3  per head: attention inside each selected chunk, fused with
//     w = softmax over the selection of scale * q_h . l_i
// (Per-token top-K retrieval over chunk landmarks: Understanding and Improving
// Length Generalization in Hierarchical Sparse Attention Models; fusion by
// retrieval scores: HiLS Attention abstract.)
//
// The landmark scan is the HBM stream (the K/V cache itself is never read
// except for the K selected chunks).  Grid = splits x (B*Hkv) blocks; each
// block scans a contiguous range of landmark rows with 16-byte streaming loads
// (a row is d elements = D/VEC lanes; a warp covers 32*16 contiguous bytes per
// load), reduces each row's partial dot products with xor-shuffles and keeps a
// warp-distributed top-K of 64-bit (score, ~index) keys.  Blocks publish their
// K best keys, take a ticket, and the last block of each (b, g) merges all
// candidates, resets the ticket and runs D3.  There is no inter-block wait.
#include "common.cuh"

namespace hsa {

constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kDecUnroll = 4;

template <typename T, typename TL, int D>
__global__ void __launch_bounds__(kDecThreads)
decode_kernel(const T *__restrict__ q, const TL *__restrict__ lm, const T *__restrict__ Kc,
              const T *__restrict__ Vc, int H, int Hkv, int64_t Lc, int S, int topk, float scale,
              int splits, uint64_t *__restrict__ cand, unsigned *__restrict__ tickets,
              T *__restrict__ O, int32_t *__restrict__ idx_out) {
    constexpr int VEC = Vec16<TL>::N;
    constexpr int LPR = D / VEC;          // lanes per landmark row
    constexpr int RPW = 32 / LPR;         // rows per warp load
    constexpr int VT = Vec16<T>::N;
    constexpr int RS = D + VT;            // padded K/V row stride in shared memory
    constexpr int R = D / 32;

    __shared__ float qbar_s[D];
    __shared__ uint64_t lists[kDecWarps][32];
    __shared__ int is_last;
    __shared__ int32_t sel_s[32];
    __shared__ float wsel[16][32];
    extern __shared__ float4 dyn4[];

    const int split = blockIdx.x;
    const int64_t bg = blockIdx.y;
    const int64_t b = bg / Hkv;
    const int g = (int)(bg % Hkv);
    const int G = H / Hkv;
    const int64_t Nc = Lc / S;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    for (int j = tid; j < D; j += kDecThreads) {
        float a = 0.f;
        for (int h = 0; h < G; ++h) a += to_f32(q[(b * H + g * G + h) * D + j]);
        qbar_s[j] = a / (float)G;
    }
    __syncthreads();

    // ---------------------------------------------------------------- D1: scan
    const int col = (lane % LPR) * VEC;
    const int sub = lane / LPR;
    float qv[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) qv[e] = qbar_s[col + e];
    const int64_t r0 = (int64_t)split * Nc / splits;
    const int64_t r1 = (int64_t)(split + 1) * Nc / splits;
    const TL *lm_bg = lm + bg * Nc * D;

    WarpTopK tk;
    tk.init(topk);
    uint64_t thr = 0ull;
    constexpr int STEP = kDecWarps * kDecUnroll * RPW;
    for (int64_t base = r0; base < r1; base += STEP) {
        uint4 raw[kDecUnroll];
#pragma unroll
        for (int u = 0; u < kDecUnroll; ++u) {
            const int64_t row = base + (int64_t)(warp * kDecUnroll + u) * RPW + sub;
            raw[u] = row < r1 ? ld_stream16(lm_bg + row * D + col) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kDecUnroll; ++u) {
            const int64_t row = base + (int64_t)(warp * kDecUnroll + u) * RPW + sub;
            float f[VEC];
            Vec16<TL>::unpack(raw[u], f);
            float a = 0.f;
#pragma unroll
            for (int e = 0; e < VEC; ++e) a = fmaf(qv[e], f[e], a);
#pragma unroll
            for (int o = LPR / 2; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
            const uint64_t key = row < r1 ? make_key(scale * a, row) : 0ull;
#pragma unroll
            for (int s = 0; s < RPW; ++s) {
                const uint64_t x = __shfl_sync(0xffffffffu, key, s * LPR);
                if (x > thr) {
                    tk.insert(x);
                    thr = tk.threshold();
                }
            }
        }
    }
    // block merge of the warp lists
    lists[warp][lane] = tk.v;
    __syncthreads();
    if (warp == 0) {
        for (int w2 = 1; w2 < kDecWarps; ++w2) {
            for (int k = 0; k < topk; ++k) {
                const uint64_t x = lists[w2][k];
                if (x > thr) {
                    tk.insert(x);
                    thr = tk.threshold();
                }
            }
        }
        if (lane < topk) cand[(bg * splits + split) * topk + lane] = tk.v;
    }

    // ---------------------------------------------------------------- D2: last block merges
    __threadfence();
    __syncthreads();
    if (tid == 0) is_last = (atomicAdd(&tickets[bg], 1u) == (unsigned)(splits - 1));
    __syncthreads();
    if (!is_last) return;
    __threadfence();

    tk.init(topk);
    thr = 0ull;
    const int64_t ncand = (int64_t)splits * topk;
    const uint64_t *cb = cand + bg * ncand;
    for (int64_t c0 = (int64_t)warp * 32; c0 < ncand; c0 += kDecThreads) {
        const uint64_t x = (c0 + lane < ncand)
            ? (uint64_t)__ldcg(reinterpret_cast<const unsigned long long *>(cb + c0 + lane)) : 0ull;
        for (int s = 0; s < 32; ++s) {
            const uint64_t y = __shfl_sync(0xffffffffu, x, s);
            if (y > thr) {
                tk.insert(y);
                thr = tk.threshold();
            }
        }
    }
    __syncthreads();
    lists[warp][lane] = tk.v;
    __syncthreads();
    if (warp == 0) {
        for (int w2 = 1; w2 < kDecWarps; ++w2) {
            for (int k = 0; k < topk; ++k) {
                const uint64_t x = lists[w2][k];
                if (x > thr) {
                    tk.insert(x);
                    thr = tk.threshold();
                }
            }
        }
        if (lane < topk) {
            const int32_t i = key_index(tk.v);
            sel_s[lane] = i;
            if (idx_out) idx_out[bg * topk + lane] = i;
        }
        if (lane == 0) tickets[bg] = 0u;        // ready for the next call
    }
    __syncthreads();

    // ---------------------------------------------------------------- D3: attend + fuse
    float *qs = reinterpret_cast<float *>(dyn4);                  // [G][D]
    T *ks = reinterpret_cast<T *>(qs + G * D);                    // [64][RS]
    T *vs = ks + 64 * RS;
    for (int e = tid; e < G * D; e += kDecThreads) qs[e] = to_f32(q[(b * H + g * G) * D + e]);
    __syncthreads();
    // fusion weights per head over the selection
    for (int h = warp; h < G; h += kDecWarps) {
        float s[32];
        float mx = -INFINITY;
        for (int k = 0; k < topk; ++k) {
            const int32_t i = sel_s[k];
            float a = 0.f;
            if (i >= 0) {
                const TL *lp = lm_bg + (int64_t)i * D;
                for (int j = lane; j < D; j += 32) a = fmaf(qs[h * D + j], to_f32(lp[j]), a);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
            s[k & 31] = i >= 0 ? scale * a : -INFINITY;
            mx = fmaxf(mx, s[k & 31]);
        }
        float den = 0.f;
        for (int k = 0; k < topk; ++k) {
            s[k] = sel_s[k] >= 0 ? expf(s[k] - mx) : 0.f;
            den += s[k];
        }
        if (lane == 0)
            for (int k = 0; k < topk; ++k) wsel[h][k] = den > 0.f ? s[k] / den : 0.f;
    }
    float acc[2][R];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh)
#pragma unroll
        for (int r = 0; r < R; ++r) acc[hh][r] = 0.f;
    const T *Kbg = Kc + bg * Lc * D;
    const T *Vbg = Vc + bg * Lc * D;
    for (int k = 0; k < topk; ++k) {
        const int32_t ci = sel_s[k];
        if (ci < 0) continue;
        __syncthreads();
        const int64_t first = (int64_t)ci * S;
        for (int e = tid; e < S * (D / VT); e += kDecThreads) {
            const int r = e / (D / VT), c = (e % (D / VT)) * VT;
            *reinterpret_cast<uint4 *>(ks + r * RS + c) = ld_stream16(Kbg + (first + r) * D + c);
            *reinterpret_cast<uint4 *>(vs + r * RS + c) = ld_stream16(Vbg + (first + r) * D + c);
        }
        __syncthreads();
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int h = warp + hh * kDecWarps;
            if (h >= G) break;
            const float *qh = qs + h * D;
            float lg[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int j = lane + 32 * u;
                float a = 0.f;
#pragma unroll 4
                for (int c = 0; c < D; c += VT) {
                    float f[VT];
                    Vec16<T>::unpack(*reinterpret_cast<const uint4 *>(ks + j * RS + c), f);
#pragma unroll
                    for (int e = 0; e < VT; ++e) a = fmaf(qh[c + e], f[e], a);
                }
                lg[u] = scale * a;
            }
            float mx = fmaxf(lg[0], lg[1]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            float p0 = expf(lg[0] - mx), p1 = expf(lg[1] - mx);
            float den = p0 + p1;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
            float o_r[R];
#pragma unroll
            for (int r = 0; r < R; ++r) o_r[r] = 0.f;
            for (int j = 0; j < 64; ++j) {
                const float pj = __shfl_sync(0xffffffffu, j < 32 ? p0 : p1, j & 31);
#pragma unroll
                for (int r = 0; r < R; ++r)
                    o_r[r] = fmaf(pj, to_f32(vs[j * RS + lane + 32 * r]), o_r[r]);
            }
            const float f = wsel[h][k] / den;
#pragma unroll
            for (int r = 0; r < R; ++r) acc[hh][r] = fmaf(f, o_r[r], acc[hh][r]);
        }
    }
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        const int h = warp + hh * kDecWarps;
        if (h >= G) break;
        T *op = O + (b * H + g * G + h) * (int64_t)D;
#pragma unroll
        for (int r = 0; r < R; ++r) op[lane + 32 * r] = from_f32<T>(acc[hh][r]);
    }
}

int decode_splits(int B, int Hkv, int64_t Nc, int num_sms) {
    const int64_t pairs = (int64_t)B * Hkv;
    int64_t s = (4LL * num_sms + pairs - 1) / pairs;
    const int64_t max_s = (Nc + 255) / 256;          // at least 256 rows per split
    if (s > max_s) s = max_s;
    if (s < 1) s = 1;
    if (s > 65535) s = 65535;
    return (int)s;
}

size_t decode_dyn_smem(int G, int d, bool bf16) {
    const int vt = bf16 ? 8 : 4;
    const size_t el = bf16 ? 2 : 4;
    return sizeof(float) * (size_t)G * d + 2 * el * 64 * (size_t)(d + vt);
}

template <typename T, typename TL, int D>
static cudaError_t launch_decode_t(const void *q, const void *lm, const void *Kc, const void *Vc,
                                   int B, int H, int Hkv, int64_t Lc, int S, int topk,
                                   float scale, int splits, uint64_t *cand, unsigned *tickets,
                                   void *O, int32_t *idx_out, cudaStream_t st) {
    const size_t smem = decode_dyn_smem(H / Hkv, D, sizeof(T) == 2);
    auto kern = decode_kernel<T, TL, D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)splits, (unsigned)(B * Hkv));
    kern<<<grid, kDecThreads, smem, st>>>((const T *)q, (const TL *)lm, (const T *)Kc,
                                          (const T *)Vc, H, Hkv, Lc, S, topk, scale, splits, cand,
                                          tickets, (T *)O, idx_out);
    return cudaGetLastError();
}

cudaError_t launch_decode(const void *q, const void *Kc, const void *Vc, bool bf16,
                          const void *lm, bool lm_bf16, int B, int H, int Hkv, int64_t Lc, int d,
                          int S, int topk, float scale, int splits, uint64_t *cand,
                          unsigned *tickets, void *O, int32_t *idx_out, cudaStream_t st) {
#define HSA_DEC(T, TL, DD) \
    return launch_decode_t<T, TL, DD>(q, lm, Kc, Vc, B, H, Hkv, Lc, S, topk, scale, splits, cand, tickets, O, idx_out, st)
    using bf = __nv_bfloat16;
    if (bf16) {
        if (lm_bf16) { if (d == 128) HSA_DEC(bf, bf, 128); HSA_DEC(bf, bf, 64); }
        if (d == 128) HSA_DEC(bf, float, 128);
        HSA_DEC(bf, float, 64);
    }
    if (lm_bf16) { if (d == 128) HSA_DEC(float, bf, 128); HSA_DEC(float, bf, 64); }
    if (d == 128) HSA_DEC(float, float, 128);
    HSA_DEC(float, float, 64);
#undef HSA_DEC
}

}  // namespace hsa
