// select.cu -- prefill chunk selection and fusion weights.
//
// For each (b, t, g): group query qbar = mean of the G heads' queries, group
// scores sbar_i = scale * qbar . l_i over the visible chunks i < floor(t/S),
// the top-K chunks by (score desc, index asc), then (when w_out is given) per
// head the fusion weights w = softmax over the selected chunks of
// scale * q_h . l_i.  The tensor-core attention path computes those logits
// itself, inside its S = Q K^T tiles, and passes w_out = NULL here.
// (Per-token top-K retrieval over chunk landmarks: Understanding and Improving
// Length Generalization in Hierarchical Sparse Attention Models, "Methodology
// in Plain English"; fusion by retrieval scores: HiLS Attention abstract.)
//
// With a retrieval interval R > 1 (one selection per R consecutive tokens,
// R divides S) the block's 64 rows are selection rows: row u serves tokens
// u*R .. u*R+R-1 and its group query is token u*R's (pool_mean = 0) or the
// mean over those tokens (pool_mean = 1); the fusion weights stay per token.
//
// One block owns 64 consecutive (selection) rows of one (b, g).  Their qbar rows stay
// in shared memory while the landmark rows of the visible chunks stream
// through shared memory 32 at a time.  Each thread scores one token against 8
// chunks of a tile (fp32 FMA, float4 operands) into a shared score tile; then
// each warp folds the tile into the sorted top-K lists of its 8 tokens, kept
// warp-distributed (lane k holds a token's k-th best 64-bit key), with
// bitonic sorting and merging networks.
#include "common.cuh"

namespace hsa {

constexpr int kSelTokens = 64;   // tokens per block
constexpr int kSelChunks = 32;   // landmark rows per shared-memory tile
constexpr int kSelThreads = 256; // 8 warps, 8 tokens per warp
constexpr int kSelTokPerWarp = kSelTokens / (kSelThreads / 32);

template <typename T, typename TL, int D>
__global__ void __launch_bounds__(kSelThreads)
select_kernel(const T *__restrict__ Q, const TL *__restrict__ lm, int H, int Hkv, int64_t L,
              int S, int64_t Nc, Chunks ch, int topk, float scale, int R, int pool_mean,
              int32_t *__restrict__ idx_out, float *__restrict__ w_out) {
    extern __shared__ float4 smem4[];
    float *qbar = reinterpret_cast<float *>(smem4);                 // [64][D+4]
    float *lmt = qbar + kSelTokens * (D + 4);                        // [32][D+4]
    float *sc = lmt + kSelChunks * (D + 4);                          // [64][33]

    const int64_t Lsel = (L + R - 1) / R;                           // selection rows
    const int n_tiles = (int)((Lsel + kSelTokens - 1) / kSelTokens);
    const int tile = n_tiles - 1 - (int)blockIdx.x;                 // heavy tiles first
    const int g = blockIdx.y, b = blockIdx.z;
    const int G = H / Hkv;
    const int64_t t0 = (int64_t)tile * kSelTokens;                  // first selection row
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // qbar for the block's tokens (rows past L are zero).  A thread owns one
    // 16-byte vector (VT elements of d) of a token and sums it over the G
    // heads; all of a thread's loads are independent, so many are in flight.
    {
        constexpr int VT = Vec16<T>::N;
        constexpr int VPR = D / VT;                          // vectors per row
        constexpr int PER = kSelTokens * VPR / kSelThreads;  // (token, vector) pairs per thread
        static_assert(PER * kSelThreads == kSelTokens * VPR, "qbar pairs must split evenly");
        float acc[PER][VT];
#pragma unroll
        for (int u = 0; u < PER; ++u)
#pragma unroll
            for (int v = 0; v < VT; ++v) acc[u][v] = 0.f;
        // (token, head) pairs of a row: the G heads of its first token, or of
        // each of its tokens (pool_mean); rows and tokens past the end add 0
        const int npairs = pool_mean ? G * R : G;
        for (int h = 0; h < npairs; ++h) {
            const int tok = h / G, hd = h % G;
            uint4 raw[PER];
#pragma unroll
            for (int u = 0; u < PER; ++u) {
                const int e = tid + u * kSelThreads, r = e / VPR, c = (e % VPR) * VT;
                const int64_t t = (t0 + r) * R + tok;
                raw[u] = (t0 + r < Lsel && t < L)
                             ? ld_stream16(Q + ((b * L + t) * H + (int64_t)g * G + hd) * D + c)
                             : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < PER; ++u) {
                float f[VT];
                Vec16<T>::unpack(raw[u], f);
#pragma unroll
                for (int v = 0; v < VT; ++v) acc[u][v] += f[v];
            }
        }
#pragma unroll
        for (int u = 0; u < PER; ++u) {
            const int e = tid + u * kSelThreads, r = e / VPR, c = (e % VPR) * VT;
            const int64_t left = L - (t0 + r) * R;
            const int n = pool_mean ? G * (int)(left < R ? (left > 0 ? left : 1) : R) : G;
            const float inv = 1.f / (float)n;
#pragma unroll
            for (int v = 0; v < VT; ++v) qbar[r * (D + 4) + c + v] = acc[u][v] * inv;
        }
    }
    const int64_t t_last = (t0 + kSelTokens - 1 < Lsel ? t0 + kSelTokens - 1 : Lsel - 1);
    const int64_t nvis_max = chunk_of(ch, t_last * R);

    // scoring role: token tok_s, chunks sub + 4m of each tile
    const int tok_s = tid >> 2, sub = tid & 3;
    // list role: this warp's tokens, each a sorted list of KP keys replicated
    // in every KP-lane segment of v[u] (lane k < topk holds the k-th best)
    const int KP = pow2_at_least(topk);
    uint64_t v[kSelTokPerWarp];
#pragma unroll
    for (int u = 0; u < kSelTokPerWarp; ++u) v[u] = 0ull;

    const TL *lm_bg = lm + ((int64_t)b * Hkv + g) * Nc * D;
    for (int64_t c0 = 0; c0 < nvis_max; c0 += kSelChunks) {
        __syncthreads();
        {
            // landmark rows c0 .. c0+31 as fp32, 16-byte loads all in flight
            constexpr int VL = Vec16<TL>::N;
            constexpr int LPT = kSelChunks * (D / VL) / kSelThreads;   // vectors per thread
            uint4 raw[LPT];
#pragma unroll
            for (int u = 0; u < LPT; ++u) {
                const int e = tid + u * kSelThreads, r = e / (D / VL), c = (e % (D / VL)) * VL;
                const int64_t i = c0 + r;
                raw[u] = i < nvis_max ? *reinterpret_cast<const uint4 *>(lm_bg + i * D + c)
                                      : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < LPT; ++u) {
                const int e = tid + u * kSelThreads, r = e / (D / VL), c = (e % (D / VL)) * VL;
                float f[VL];
                Vec16<TL>::unpack(raw[u], f);
#pragma unroll
                for (int v = 0; v < VL; ++v) lmt[r * (D + 4) + c + v] = f[v];
            }
        }
        __syncthreads();
        {
            float acc[8];
#pragma unroll
            for (int m = 0; m < 8; ++m) acc[m] = 0.f;
            const float4 *qv = reinterpret_cast<const float4 *>(qbar + tok_s * (D + 4));
#pragma unroll 4
            for (int j4 = 0; j4 < D / 4; ++j4) {
                const float4 a = qv[j4];
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    const float4 l =
                        reinterpret_cast<const float4 *>(lmt + (sub + 4 * m) * (D + 4))[j4];
                    acc[m] = fmaf(a.x, l.x, acc[m]);
                    acc[m] = fmaf(a.y, l.y, acc[m]);
                    acc[m] = fmaf(a.z, l.z, acc[m]);
                    acc[m] = fmaf(a.w, l.w, acc[m]);
                }
            }
#pragma unroll
            for (int m = 0; m < 8; ++m) sc[tok_s * 33 + sub + 4 * m] = scale * acc[m];
        }
        __syncthreads();
        // fold the tile into each token's top-KP list: bitonic-sort the 32
        // keys into KP-long runs, merge the runs, merge into the running list
        // (the warp's 8 tokens are independent chains of shuffles)
#pragma unroll
        for (int u = 0; u < kSelTokPerWarp; ++u) {
            const int tok = warp * kSelTokPerWarp + u;
            const int64_t t = t0 + tok;                              // selection row
            const int64_t nvis = t < Lsel ? chunk_of(ch, t * R) : 0;
            const int64_t i = c0 + lane;
            const uint64_t key = i < nvis ? make_key(sc[tok * 33 + lane], i) : 0ull;
            v[u] = merge_lists(v[u], merge_segments(sort_segments_desc(key, KP), KP), KP);
        }
    }

    // outputs: idx (lane k = rank k) and per-head fusion weights.  For the
    // logits the warp is split into KP slots (KP = topk rounded up to a power
    // of two) of PARTS = 32/KP lanes; the lanes of slot k split d and reduce
    // with PARTS-wide shuffles, so all slots of a head are computed at once.
    const int PARTS = 32 / KP;
    const int slot = lane / PARTS, part = lane % PARTS;
    const int span = D / PARTS;                       // d elements per lane
#pragma unroll 1
    for (int u = 0; u < kSelTokPerWarp; ++u) {
        const int64_t row = t0 + warp * kSelTokPerWarp + u;
        if (row >= Lsel) continue;
        const int32_t sel = lane < topk ? key_index(v[u]) : -1;
        const int32_t my_sel = __shfl_sync(0xffffffffu, sel, slot < 32 ? slot : 0);
        const bool active = slot < topk && my_sel >= 0;
        const TL *lp = lm_bg + (int64_t)(my_sel > 0 ? my_sel : 0) * D + part * span;
        // the row's selection serves its R tokens; the weights are per token
#pragma unroll 1
        for (int j = 0; j < R; ++j) {
        const int64_t t = row * R + j;
        if (t >= L) break;
        if (lane < topk && idx_out) idx_out[((b * L + t) * Hkv + g) * topk + lane] = sel;
        if (w_out == nullptr) continue;     // weights computed downstream (tensor-core path)
#pragma unroll 1
        for (int h = 0; h < G; ++h) {
            const int hh = g * G + h;
            const T *qh = Q + ((b * L + t) * H + hh) * (int64_t)D + part * span;
            float a = 0.f;
            if (active) {
#pragma unroll 4
                for (int e = 0; e < span; ++e) a = fmaf(to_f32(qh[e]), to_f32(lp[e]), a);
            }
            for (int o = PARTS / 2; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
            const float s = active ? scale * a : -INFINITY;
            float mx = s;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            const float e = (active && part == 0) ? expf(s - mx) : 0.f;
            float den = e;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
            if (part == 0 && slot < topk)
                w_out[((b * L + t) * H + hh) * topk + slot] = (active && den > 0.f) ? e / den : 0.f;
        }
        }
    }
}

template <typename T, typename TL, int D>
static cudaError_t launch_select_t(const void *Q, const void *lm, int B, int H, int Hkv,
                                   int64_t L, int S, int64_t Nc, Chunks ch, int topk, float scale,
                                   int R, int pool_mean, int32_t *idx, float *w, cudaStream_t st) {
    const size_t smem =
        sizeof(float) * ((kSelTokens + kSelChunks) * (D + 4) + kSelTokens * 33);
    auto kern = select_kernel<T, TL, D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t Lsel = (L + R - 1) / R;
    dim3 grid((unsigned)((Lsel + kSelTokens - 1) / kSelTokens), (unsigned)Hkv, (unsigned)B);
    kern<<<grid, kSelThreads, smem, st>>>((const T *)Q, (const TL *)lm, H, Hkv, L, S, Nc, ch,
                                          topk, scale, R, pool_mean, idx, w);
    return cudaGetLastError();
}

template <typename T, typename TL>
static cudaError_t launch_select_l(const void *Q, const void *lm, int B, int H, int Hkv,
                                   int64_t L, int d, int S, int64_t Nc, Chunks ch, int topk,
                                   float scale, int R, int pool_mean, int32_t *idx, float *w,
                                   cudaStream_t st) {
    return d == 128 ? launch_select_t<T, TL, 128>(Q, lm, B, H, Hkv, L, S, Nc, ch, topk, scale, R, pool_mean, idx, w, st)
                    : launch_select_t<T, TL, 64>(Q, lm, B, H, Hkv, L, S, Nc, ch, topk, scale, R, pool_mean, idx, w, st);
}

// Nc: chunks with a landmark (L / S, or the number of variable-length chunks
// given by bounds / tok_chunk, both null for chunks of S tokens).
cudaError_t launch_select(const void *Q, bool q_bf16, const void *lm, bool lm_bf16, int B, int H,
                          int Hkv, int64_t L, int d, int S, int64_t Nc, const int32_t *bounds,
                          const int32_t *tok_chunk, int topk, float scale, int R, int pool_mean,
                          int32_t *idx, float *w, cudaStream_t st) {
    using bf = __nv_bfloat16;
    const Chunks ch = {bounds, tok_chunk, L, S};
    if (q_bf16)
        return lm_bf16 ? launch_select_l<bf, bf>(Q, lm, B, H, Hkv, L, d, S, Nc, ch, topk, scale, R, pool_mean, idx, w, st)
                       : launch_select_l<bf, float>(Q, lm, B, H, Hkv, L, d, S, Nc, ch, topk, scale, R, pool_mean, idx, w, st);
    return lm_bf16 ? launch_select_l<float, bf>(Q, lm, B, H, Hkv, L, d, S, Nc, ch, topk, scale, R, pool_mean, idx, w, st)
                   : launch_select_l<float, float>(Q, lm, B, H, Hkv, L, d, S, Nc, ch, topk, scale, R, pool_mean, idx, w, st);
}

}  // namespace hsa
