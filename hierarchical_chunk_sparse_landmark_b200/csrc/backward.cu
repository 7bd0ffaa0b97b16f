// backward.cu -- gradients of the prefill on CUDA cores (fp32 accumulate).
//
// HiLS Attention abstract: the retrieval scores are trained end to end with
// the language-model loss, so the gradient of O reaches the queries, the keys
// and values of the retrieved chunks, and the landmarks through the fusion
// weights.  The selection is a hard top-K and is held fixed (the forward's
// indices are an input).  Per query row (t, h) of KV group g with selected
// chunks i_1 .. i_K (HSA "Methodology in Plain English"):
//
//   z_k = scale q.l_{i_k}, w = softmax(z);  p_k = softmax_j(scale q.k_j), o_k = p_k V
//   O = sum_k w_k o_k + own-chunk term (weight 1)
//   u_kj = dO.v_j, dw_k = p_k.u_k (= dO.o_k), dz_k = w_k (dw_k - sum_k' w_k' dw_k')
//   da_kj = w_k p_kj (u_kj - dw_k)            (own chunk: w = 1)
//   dq   = scale (sum_kj da_kj k_j + sum_k dz_k l_{i_k})
//   dk_j += scale da_kj q,  dv_j += w_k p_kj dO,  dl_{i_k} += scale dz_k q
//   DHSA landmarks (sqrt(S) * mean of the chunk's keys): dk_j += dl / sqrt(S).
//
// Four steps, all deterministic (no floating-point atomics):
//   bwd_row_kernel    row-centric: dQ and the per-slot (w_k, dz_k), one block
//                     per (b, t, g), one warp per query head (two passes over
//                     the selected chunks: dw_k first, then dq)
//   hist/scan/scatter a stable counting sort of the valid selection entries
//                     by (b, g, chunk), in (t, slot) order, cut into segments
//                     of at most kSegRows query rows (plus one own-chunk
//                     segment per chunk)
//   bwd_key_kernel    key-centric: one block per segment recomputes the chunk
//                     softmax of its rows and accumulates dK, dV (64 x d) and
//                     dl (d) of its chunk in registers -> per-segment partials
//   bwd_reduce_kernel sums each chunk's partials in segment order into dK, dV
//                     (every row written once) and the landmark gradient
#include <cuda_fp16.h>

#include "common.cuh"

namespace hsa {

constexpr int kSegRows = 1024;          // query rows (entry x head) per key segment
constexpr int kKeyThreads = 512;        // 64 keys x 8 lanes over d
constexpr int kKeyLanes = kKeyThreads / 64;
constexpr int kScanThreads2 = 1024;

// A selection entry counts when it names a chunk before the token's own chunk
// (and one with a landmark); anything else is flagged and skipped.
__device__ __forceinline__ bool sel_ok(int32_t ci, int64_t t, int S, int64_t Nc) {
    return ci >= 0 && (int64_t)ci < Nc && (int64_t)ci < t / S;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float lm_at(const void *lm, int lm_bf16, int64_t i) {
    return lm_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(lm)[i])
                   : reinterpret_cast<const float *>(lm)[i];
}

// ---------------------------------------------------------------- row-centric
// One pass over the selected chunks: the fusion weights depend only on q and
// the landmarks, so they come first; then every chunk is staged once and its
// dw_k and da_k (hence its dq terms) follow from its own softmax.
template <typename T, int D>
__global__ void __launch_bounds__(512)
bwd_row_kernel(const T *__restrict__ Q, const T *__restrict__ K, const T *__restrict__ V,
               const void *__restrict__ lm, int lm_bf16, const int32_t *__restrict__ idx,
               const T *__restrict__ dO, int H, int Hkv, int64_t L, int S, int64_t Nc, int topk,
               int own_chunk, float scale, float2 *__restrict__ coef, float *__restrict__ dQ,
               unsigned *__restrict__ status) {
    constexpr int VEC = Vec16<T>::N;
    constexpr int RS = D + VEC;                   // padded row stride of the K/V stage
    constexpr int R = D / 32;                     // d elements per lane
    extern __shared__ float4 smem4[];
    const int G = H / Hkv;
    float *qs = reinterpret_cast<float *>(smem4);                  // [G][D]
    float *dos = qs + G * D;                                       // [G][D]
    T *ks = reinterpret_cast<T *>(dos + G * D);                    // [64][RS]
    T *vs = ks + 64 * RS;                                          // [64][RS]

    const int64_t t = blockIdx.x;
    const int g = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nthr = blockDim.x;
    const int64_t row = (int64_t)b * L + t;
    for (int e = threadIdx.x; e < G * D; e += nthr) {
        qs[e] = to_f32(Q[(row * H + (int64_t)g * G) * D + e]);
        dos[e] = to_f32(dO[(row * H + (int64_t)g * G) * D + e]);
    }
    __syncthreads();
    const int64_t bg = (int64_t)b * Hkv + g;
    const T *Kbg = K + bg * L * D;
    const T *Vbg = V + bg * L * D;
    const int32_t *ip = idx + (row * Hkv + g) * topk;
    const int h = g * G + warp;
    const float *qh = qs + warp * D, *doh = dos + warp * D;
    const int64_t c_t = t / S;

    // fusion logits z_k = scale q.l_{i_k} and weights w = softmax over the
    // valid slots (lane k keeps slot k)
    float zk = -INFINITY;
    bool vk = false;
    for (int it = 0; it < topk; ++it) {
        const int32_t ci = ip[it];
        if (!sel_ok(ci, t, S, Nc)) {
            if (ci >= 0 && threadIdx.x == 0) atomicOr(status, kFlagBadIdx);
            continue;
        }
        float a = 0.f;
#pragma unroll
        for (int r = 0; r < R; ++r)
            a = fmaf(qh[lane + 32 * r], lm_at(lm, lm_bf16, (bg * Nc + ci) * D + lane + 32 * r), a);
        const float z = scale * warp_sum(a);
        if (lane == it) { zk = z; vk = true; }
    }
    const float m = warp_max(vk ? zk : -INFINITY);
    const float ew = vk ? expf(zk - m) : 0.f;
    const float sw = warp_sum(ew);
    const float wk = vk ? ew / sw : 0.f;

    float dq[R];
#pragma unroll
    for (int r = 0; r < R; ++r) dq[r] = 0.f;
    float dwk = 0.f;
    const int n_items = topk + (own_chunk ? 1 : 0);
    for (int it = 0; it < n_items; ++it) {
        int64_t first;
        int nk;
        if (it < topk) {
            const int32_t ci = ip[it];
            if (!sel_ok(ci, t, S, Nc)) continue;   // uniform across the block
            first = (int64_t)ci * S;
            nk = S;
        } else {
            first = c_t * S;
            nk = (int)(t - first + 1);
        }
        __syncthreads();
        const int vpr = D / VEC;
        for (int e = threadIdx.x; e < nk * vpr; e += nthr) {
            const int r = e / vpr, c = (e % vpr) * VEC;
            *reinterpret_cast<uint4 *>(ks + r * RS + c) =
                *reinterpret_cast<const uint4 *>(Kbg + (first + r) * D + c);
            *reinterpret_cast<uint4 *>(vs + r * RS + c) =
                *reinterpret_cast<const uint4 *>(Vbg + (first + r) * D + c);
        }
        __syncthreads();
        // keys j = lane, lane + 32: s_j = scale q.k_j, u_j = dO.v_j
        float sj[2], uj[2];
#pragma unroll
        for (int w2 = 0; w2 < 2; ++w2) {
            const int j = lane + 32 * w2;
            sj[w2] = -INFINITY;
            uj[w2] = 0.f;
            if (j < nk) {
                float a = 0.f, c = 0.f;
#pragma unroll 4
                for (int x = 0; x < D; x += VEC) {
                    float fk[VEC], fv[VEC];
                    Vec16<T>::unpack(*reinterpret_cast<const uint4 *>(ks + j * RS + x), fk);
                    Vec16<T>::unpack(*reinterpret_cast<const uint4 *>(vs + j * RS + x), fv);
#pragma unroll
                    for (int e = 0; e < VEC; ++e) {
                        a = fmaf(qh[x + e], fk[e], a);
                        c = fmaf(doh[x + e], fv[e], c);
                    }
                }
                sj[w2] = scale * a;
                uj[w2] = c;
            }
        }
        const float mx = warp_max(fmaxf(sj[0], sj[1]));
        float p[2];
#pragma unroll
        for (int w2 = 0; w2 < 2; ++w2) p[w2] = lane + 32 * w2 < nk ? expf(sj[w2] - mx) : 0.f;
        const float inv = 1.f / warp_sum(p[0] + p[1]);
        p[0] *= inv;
        p[1] *= inv;
        const float dw = warp_sum(p[0] * uj[0] + p[1] * uj[1]);
        const float a = it < topk ? __shfl_sync(0xffffffffu, wk, it) : 1.f;
        if (it < topk && lane == it) dwk = dw;
        float da[2];
#pragma unroll
        for (int w2 = 0; w2 < 2; ++w2) da[w2] = scale * a * p[w2] * (uj[w2] - dw);
        for (int j = 0; j < nk; ++j) {
            const float dj = __shfl_sync(0xffffffffu, da[j >> 5], j & 31);
#pragma unroll
            for (int r = 0; r < R; ++r) dq[r] = fmaf(dj, to_f32(ks[j * RS + lane + 32 * r]), dq[r]);
        }
    }
    // dz = w (dw - sum w dw); dq += scale sum_k dz_k l_k
    const float dsum = warp_sum(wk * dwk);
    const float dzk = wk * (dwk - dsum);
    if (lane < topk) coef[(row * H + h) * topk + lane] = make_float2(wk, dzk);
    for (int it = 0; it < topk; ++it) {
        const int32_t ci = ip[it];
        if (!sel_ok(ci, t, S, Nc)) continue;
        const float dz = scale * __shfl_sync(0xffffffffu, dzk, it);
#pragma unroll
        for (int r = 0; r < R; ++r)
            dq[r] = fmaf(dz, lm_at(lm, lm_bf16, (bg * Nc + ci) * D + lane + 32 * r), dq[r]);
    }
    float *dqh = dQ + (row * H + h) * (int64_t)D;
#pragma unroll
    for (int r = 0; r < R; ++r) dqh[lane + 32 * r] = dq[r];
}

// ---------------------------------------------------------------- entry lists
// cnt[((bg * Nc) + c) * NTB + tb] = valid entries of token block tb of (b, g)
// that selected chunk c (the matrix is zeroed first).
__global__ void __launch_bounds__(256)
bwd_hist_kernel(const int32_t *__restrict__ idx, int Hkv, int64_t L, int S, int64_t Nc, int topk,
                int64_t TB, int64_t NTB, int use_smem, int32_t *__restrict__ cnt) {
    extern __shared__ int32_t hist[];
    const int64_t bg = blockIdx.y, tb = blockIdx.x;
    const int64_t b = bg / Hkv, g = bg % Hkv;
    if (use_smem) {
        for (int64_t c = threadIdx.x; c < Nc; c += blockDim.x) hist[c] = 0;
        __syncthreads();
    }
    const int64_t t0 = tb * TB;
    const int64_t n = (t0 + TB < L ? TB : L - t0) * topk;
    for (int64_t e = threadIdx.x; e < n; e += blockDim.x) {
        const int64_t t = t0 + e / topk;
        const int k = (int)(e % topk);
        const int32_t ci = idx[((b * L + t) * Hkv + g) * topk + k];
        if (!sel_ok(ci, t, S, Nc)) continue;
        if (use_smem) atomicAdd(&hist[ci], 1);
        else atomicAdd(&cnt[(bg * Nc + ci) * NTB + tb], 1);
    }
    if (use_smem) {
        __syncthreads();
        for (int64_t c = threadIdx.x; c < Nc; c += blockDim.x) cnt[(bg * Nc + c) * NTB + tb] = hist[c];
    }
}

// Block-wide exclusive scan of one value per thread (kScanThreads2 threads).
__device__ __forceinline__ int64_t block_exscan(int64_t v, int64_t *warp_tot, int64_t &total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int64_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int64_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int64_t wt = lane < (int)(blockDim.x >> 5) ? warp_tot[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int64_t y = __shfl_up_sync(0xffffffffu, wt, o);
            if (lane >= o) wt += y;
        }
        warp_tot[lane] = wt;                       // inclusive warp prefix
    }
    __syncthreads();
    const int64_t before = warp > 0 ? warp_tot[warp - 1] : 0;
    total = warp_tot[(blockDim.x >> 5) - 1];
    __syncthreads();
    return before + x - v;
}

// One block.  (1) cnt -> exclusive offsets over (bg, c, tb): the entries of
// chunk (bg, c) start at cnt[(bg*Nc + c)*NTB] in the sorted list.  (2) the
// segments: per chunk id q = bg*NcAll + c, one own-chunk segment (own_chunk)
// and ceil(n_c / E) entry segments; seg = {q, first entry, entries, own}.
__global__ void __launch_bounds__(kScanThreads2)
bwd_scan_kernel(int32_t *__restrict__ cnt, int64_t BG, int64_t Nc, int64_t NcAll, int64_t NTB,
                int own_chunk, int E, int4 *__restrict__ segs, int32_t *__restrict__ nseg,
                int32_t *__restrict__ chunk_seg_beg, int32_t *__restrict__ chunk_nseg) {
    __shared__ int64_t warp_tot[32];
    const int64_t M = BG * Nc * NTB;
    constexpr int ITEMS = 8;
    int64_t carry = 0;
    for (int64_t base = 0; base < M; base += (int64_t)kScanThreads2 * ITEMS) {
        const int64_t i0 = base + (int64_t)threadIdx.x * ITEMS;
        int32_t v[ITEMS];
        int64_t s = 0;
#pragma unroll
        for (int i = 0; i < ITEMS; ++i) {
            v[i] = i0 + i < M ? cnt[i0 + i] : 0;
            s += v[i];
        }
        int64_t total;
        int64_t run = carry + block_exscan(s, warp_tot, total);
#pragma unroll
        for (int i = 0; i < ITEMS; ++i) {
            if (i0 + i < M) cnt[i0 + i] = (int32_t)run;
            run += v[i];
        }
        carry += total;
    }
    __syncthreads();
    const int64_t n_entries = carry;
    // segments per chunk id
    const int64_t NQ = BG * NcAll;
    int64_t seg_carry = 0;
    for (int64_t base = 0; base < NQ; base += kScanThreads2) {
        const int64_t q = base + threadIdx.x;
        int64_t beg = 0, n = 0, ns = 0;
        if (q < NQ) {
            const int64_t bg = q / NcAll, c = q % NcAll;
            if (c < Nc) {
                const int64_t cell = (bg * Nc + c) * NTB;
                beg = cnt[cell];
                const int64_t end = cell + NTB < M ? cnt[cell + NTB] : n_entries;
                n = end - beg;
            }
            ns = (own_chunk ? 1 : 0) + (n + E - 1) / E;
        }
        int64_t total;
        const int64_t sb = seg_carry + block_exscan(ns, warp_tot, total);
        if (q < NQ) {
            chunk_seg_beg[q] = (int32_t)sb;
            chunk_nseg[q] = (int32_t)ns;
            int64_t s = sb;
            if (own_chunk) segs[s++] = make_int4((int)q, 0, 0, 1);
            for (int64_t e = 0; e < n; e += E)
                segs[s++] = make_int4((int)q, (int)(beg + e), (int)(n - e < E ? n - e : E), 0);
        }
        seg_carry += total;
    }
    if (threadIdx.x == 0) *nseg = (int32_t)seg_carry;
}

// Stable scatter of the entry codes t*32 + slot into the sorted list: one warp
// per (token block, bg) walks its entries in (t, slot) order, 32 at a time;
// entries of one chunk take consecutive places after those of earlier rounds.
// The cursors of a (bg, c, tb) cell belong to this warp alone.
__global__ void __launch_bounds__(32)
bwd_scatter_kernel(const int32_t *__restrict__ idx, int Hkv, int64_t L, int S, int64_t Nc,
                   int topk, int64_t TB, int64_t NTB, int use_smem, int32_t *__restrict__ off,
                   int32_t *__restrict__ entries) {
    extern __shared__ int32_t cur[];
    const int lane = threadIdx.x;
    const int64_t bg = blockIdx.y, tb = blockIdx.x;
    const int64_t b = bg / Hkv, g = bg % Hkv;
    if (use_smem) {
        for (int64_t c = lane; c < Nc; c += 32) cur[c] = off[(bg * Nc + c) * NTB + tb];
        __syncwarp();
    }
    const int64_t t0 = tb * TB;
    const int64_t n = (t0 + TB < L ? TB : L - t0) * topk;
    for (int64_t e0 = 0; e0 < n; e0 += 32) {
        const int64_t e = e0 + lane;
        const int64_t t = t0 + e / topk;
        const int k = (int)(e % topk);
        const int32_t ci = e < n ? idx[((b * L + t) * Hkv + g) * topk + k] : -1;
        const bool ok = e < n && sel_ok(ci, t, S, Nc);
        const int key = ok ? ci : -1 - lane;       // invalid entries match nobody
        const unsigned m = __match_any_sync(0xffffffffu, key);
        const int rank = __popc(m & ((1u << lane) - 1u));
        int32_t *cp = ok ? (use_smem ? &cur[ci] : &off[(bg * Nc + ci) * NTB + tb]) : nullptr;
        const int32_t base = ok ? *cp : 0;
        __syncwarp();
        if (ok && rank == 0) *cp = base + __popc(m);
        __syncwarp();
        if (ok) entries[base + rank] = (int32_t)(t * 32 + k);
    }
}

// ---------------------------------------------------------------- key-centric
// One block per segment; thread (key j = tid / 8, lane part qd = tid % 8) owns
// the d elements qd, qd + 8, qd + 16, ... of key j's dK and dV.  Key rows are
// staged with a stride of D + 8 floats, so the 32 lanes of a warp (4 keys x 8
// parts) read 32 different banks; a row element is read by the 4 lanes of one
// part at once (a broadcast).  Rows (entry, head) go 8 at a time: scores and
// u over the thread's part, summed across the 8 parts, then the chunk softmax
// of each row across the block.
template <typename T, int D>
__global__ void __launch_bounds__(kKeyThreads, 1)
bwd_key_kernel(const T *__restrict__ Q, const T *__restrict__ K, const T *__restrict__ V,
               const T *__restrict__ dO, const float2 *__restrict__ coef,
               const int32_t *__restrict__ entries, const int4 *__restrict__ segs,
               const int32_t *__restrict__ nseg_p, int H, int Hkv, int64_t L, int S,
               int64_t NcAll, int topk, float scale, float *__restrict__ part) {
    constexpr int X = D / kKeyLanes;
    constexpr int KS = D + kKeyLanes;              // staged key row stride (floats)
    constexpr int NW = kKeyThreads / 32;
    constexpr int NR = 8;                          // rows per batch
    constexpr int VEC = Vec16<T>::N;
    const int64_t sidx = blockIdx.x;
    if (sidx >= *nseg_p) return;
    extern __shared__ float4 smem4[];
    float *Ks = reinterpret_cast<float *>(smem4);  // [64][KS]
    float *Vs = Ks + 64 * KS;                      // [64][KS]
    float *qr = Vs + 64 * KS;                      // [NR][D]
    float *dor = qr + NR * D;                      // [NR][D]
    float *red = dor + NR * D;                     // [3][NW][NR]
    __shared__ int64_t rt[NR];
    __shared__ int rh[NR], rnk[NR];
    __shared__ float rw[NR], rdz[NR];

    const int4 sg = segs[sidx];
    const int64_t q = sg.x;
    const int64_t bg = q / NcAll, c = q % NcAll;
    const int64_t b = bg / Hkv, g = bg % Hkv;
    const int G = H / Hkv;
    const int own = sg.w;
    const int64_t first = c * S;
    const int nkc = (int)(L - first < S ? L - first : S);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int i = tid; i < 64 * (D / VEC); i += kKeyThreads) {
        const int j = i / (D / VEC), x = (i % (D / VEC)) * VEC;
        float fk[VEC], fv[VEC];
        if (j < nkc) {
            Vec16<T>::unpack(*reinterpret_cast<const uint4 *>(K + (bg * L + first + j) * D + x), fk);
            Vec16<T>::unpack(*reinterpret_cast<const uint4 *>(V + (bg * L + first + j) * D + x), fv);
        } else {
#pragma unroll
            for (int e = 0; e < VEC; ++e) fk[e] = fv[e] = 0.f;
        }
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            Ks[j * KS + x + e] = fk[e];
            Vs[j * KS + x + e] = fv[e];
        }
    }
    const int j = tid / kKeyLanes, qd = tid % kKeyLanes;
    const float *kj = Ks + j * KS + qd, *vj = Vs + j * KS + qd;
    float dk[X], dv[X], dl = 0.f;
#pragma unroll
    for (int x = 0; x < X; ++x) dk[x] = dv[x] = 0.f;
    const int64_t rows = own ? (int64_t)nkc * G : (int64_t)sg.z * G;
    for (int64_t r0 = 0; r0 < rows; r0 += NR) {
        __syncthreads();                           // the previous batch's rows are consumed
        if (tid < NR) {
            const int64_t ri = r0 + tid;
            int64_t t = -1;
            int hh = 0, nk = 64;
            float w = 0.f, dz = 0.f;
            if (ri < rows) {
                const int64_t e = ri / G;
                hh = (int)(ri % G);
                if (own) {
                    t = first + e;
                    w = 1.f;
                    nk = (int)e + 1;               // causal: keys first .. t
                } else {
                    const int32_t code = entries[sg.y + e];
                    t = code >> 5;
                    const float2 cf = coef[((b * L + t) * H + g * G + hh) * topk + (code & 31)];
                    w = cf.x;
                    dz = cf.y;
                }
            }
            rt[tid] = t; rh[tid] = hh; rnk[tid] = nk; rw[tid] = w; rdz[tid] = dz;
        }
        __syncthreads();
        for (int i = tid; i < NR * (D / VEC); i += kKeyThreads) {
            const int r = i / (D / VEC), x = (i % (D / VEC)) * VEC;
            const int64_t t = rt[r];
            float fq[VEC], fo[VEC];
            if (t >= 0) {
                const int64_t off = ((b * L + t) * H + g * G + rh[r]) * D + x;
                Vec16<T>::unpack(*reinterpret_cast<const uint4 *>(Q + off), fq);
                Vec16<T>::unpack(*reinterpret_cast<const uint4 *>(dO + off), fo);
            } else {
#pragma unroll
                for (int e = 0; e < VEC; ++e) fq[e] = fo[e] = 0.f;
            }
#pragma unroll
            for (int e = 0; e < VEC; ++e) {
                qr[r * D + x + e] = fq[e];
                dor[r * D + x + e] = fo[e];
            }
        }
        __syncthreads();
        float s[NR], u[NR];
#pragma unroll
        for (int r = 0; r < NR; ++r) s[r] = u[r] = 0.f;
        // d outer, rows inner: the 2 x NR partial sums and one key / value
        // element are all that is live
#pragma unroll
        for (int x = 0; x < X; ++x) {
            const float kx = kj[kKeyLanes * x], vx = vj[kKeyLanes * x];
#pragma unroll
            for (int r = 0; r < NR; ++r) {
                s[r] = fmaf(qr[r * D + qd + kKeyLanes * x], kx, s[r]);
                u[r] = fmaf(dor[r * D + qd + kKeyLanes * x], vx, u[r]);
            }
            asm volatile("" ::: "memory");   // keep each step's loads in its step (registers)
        }
#pragma unroll
        for (int r = 0; r < NR; ++r) {
#pragma unroll
            for (int o = 1; o < kKeyLanes; o <<= 1) {
                s[r] += __shfl_xor_sync(0xffffffffu, s[r], o);
                u[r] += __shfl_xor_sync(0xffffffffu, u[r], o);
            }
            s[r] = j < rnk[r] ? scale * s[r] : -INFINITY;
        }
        // block-wide softmax of each row over the 64 keys
#pragma unroll
        for (int r = 0; r < NR; ++r) {
            float m = s[r];
#pragma unroll
            for (int o = kKeyLanes; o < 32; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if (lane == 0) red[warp * NR + r] = m;
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < NR; ++r) {
            float m = red[r];
#pragma unroll
            for (int w2 = 1; w2 < NW; ++w2) m = fmaxf(m, red[w2 * NR + r]);
            asm volatile("" ::: "memory");   // one row's loads at a time (registers)
            s[r] = j < rnk[r] ? expf(s[r] - m) : 0.f;       // s now holds e = exp(s - max)
            float z = s[r], zu = s[r] * u[r];
#pragma unroll
            for (int o = kKeyLanes; o < 32; o <<= 1) {
                z += __shfl_xor_sync(0xffffffffu, z, o);
                zu += __shfl_xor_sync(0xffffffffu, zu, o);
            }
            // lanes kKeyLanes apart hold the warp's keys of one part: lane 0
            // has the warp's sums, one term per key
            if (lane == 0) {
                red[(NW + warp) * NR + r] = z;
                red[(2 * NW + warp) * NR + r] = zu;
            }
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < NR; ++r) {
            float z = 0.f, zu = 0.f;
#pragma unroll
            for (int w2 = 0; w2 < NW; ++w2) {
                z += red[(NW + w2) * NR + r];
                zu += red[(2 * NW + w2) * NR + r];
            }
            asm volatile("" ::: "memory");
            const float p = s[r] / z, dw = zu / z;
            s[r] = scale * rw[r] * p * (u[r] - dw);          // da
            u[r] = rw[r] * p;                                // w p
        }
#pragma unroll
        for (int x = 0; x < X; ++x) {
            float a = dk[x], v = dv[x];
#pragma unroll
            for (int r = 0; r < NR; ++r) {
                a = fmaf(s[r], qr[r * D + qd + kKeyLanes * x], a);
                v = fmaf(u[r], dor[r * D + qd + kKeyLanes * x], v);
            }
            dk[x] = a;
            dv[x] = v;
            asm volatile("" ::: "memory");
        }
        if (!own && tid < D) {
#pragma unroll
            for (int r = 0; r < NR; ++r) dl = fmaf(scale * rdz[r], qr[r * D + tid], dl);
        }
    }
    float *pk = part + sidx * (int64_t)(129 * D);
#pragma unroll
    for (int x = 0; x < X; ++x) {
        pk[j * D + qd + kKeyLanes * x] = dk[x];
        pk[64 * D + j * D + qd + kKeyLanes * x] = dv[x];
    }
    if (tid < D) pk[128 * D + tid] = dl;
}

// Sums each chunk's segment partials in segment order: dK, dV rows of the
// chunk (every row of the output written once, zeros where nothing
// contributed), the landmark gradient (dlm) or, for DHSA landmarks, dl / sqrt(S)
// folded into every key of the chunk.  Grid: chunks x kReduceSlices; a block
// takes a slice of the chunk's 16-byte groups of key elements, so a chunk with
// many segments (one selected by most tokens) spreads over several SMs.
constexpr int kReduceSlices = 8;
template <int D>
__global__ void __launch_bounds__(256)
bwd_reduce_kernel(const float *__restrict__ part, const int32_t *__restrict__ chunk_seg_beg,
                  const int32_t *__restrict__ chunk_nseg, int64_t L, int S, int64_t Nc,
                  int64_t NcAll, int dhsa, float *__restrict__ dK, float *__restrict__ dV,
                  float *__restrict__ dlm) {
    __shared__ float dls[D];
    const int64_t q = blockIdx.x;
    const int64_t bg = q / NcAll, c = q % NcAll;
    const int64_t first = c * S;
    const int nkc = (int)(L - first < S ? L - first : S);
    const int64_t sb = chunk_seg_beg[q];
    const int ns = chunk_nseg[q];
    const int tid = threadIdx.x;
    if (tid < D) {
        float a = 0.f;
        for (int s = 0; s < ns; ++s) a += part[(sb + s) * (int64_t)(129 * D) + 128 * D + tid];
        dls[tid] = a;
        if (blockIdx.y == 0 && !dhsa && c < Nc) dlm[(bg * Nc + c) * D + tid] = a;
    }
    __syncthreads();
    const float fold = (dhsa && c < Nc) ? rsqrtf((float)S) : 0.f;
    const int n4 = nkc * D / 4;
    float4 *dk4 = reinterpret_cast<float4 *>(dK + (bg * L + first) * D);
    float4 *dv4 = reinterpret_cast<float4 *>(dV + (bg * L + first) * D);
    for (int i4 = blockIdx.y * blockDim.x + tid; i4 < n4; i4 += kReduceSlices * blockDim.x) {
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f), v = a;
#pragma unroll 4
        for (int s = 0; s < ns; ++s) {
            const float4 *pk = reinterpret_cast<const float4 *>(part + (sb + s) * (int64_t)(129 * D));
            const float4 x = pk[i4], y = pk[16 * D + i4];
            a.x += x.x; a.y += x.y; a.z += x.z; a.w += x.w;
            v.x += y.x; v.y += y.y; v.z += y.z; v.w += y.w;
        }
        const int col = (4 * i4) % D;
        a.x = fmaf(fold, dls[col], a.x);
        a.y = fmaf(fold, dls[col + 1], a.y);
        a.z = fmaf(fold, dls[col + 2], a.z);
        a.w = fmaf(fold, dls[col + 3], a.w);
        dk4[i4] = a;
        dv4[i4] = v;
    }
}

// ---------------------------------------------------------------- host side
cudaError_t launch_backward_tc(const void *Q, const void *K, const void *V, const void *dO,
                               const void *lm, bool lm_bf16, const int32_t *idx, int B, int H,
                               int Hkv, int64_t L, int S, int64_t Nc, int64_t NcAll, int topk,
                               int own_chunk, float scale, float2 *coef, float *dw, __half *dqp,
                               const int4 *segs, const int32_t *nseg, const int32_t *entries,
                               float *part, int64_t max_seg, unsigned *status, float *dQ,
                               int phase, cudaStream_t st);

BwdLayout bwd_layout(int B, int H, int Hkv, int64_t L, int d, int S, int topk, bool dhsa,
                     bool tc) {
    BwdLayout p;
    p.tc = tc;
    const int G = H / Hkv;
    p.BG = (int64_t)B * Hkv;
    p.Nc = L / S;
    p.NcAll = (L + S - 1) / S;
    // token blocks of the stable scatter: about 256 warps over the (b, g) pairs,
    // at least 64 tokens each, the count matrix BG x Nc x NTB kept small for
    // the one-block scan
    int64_t ntb = (256 + p.BG - 1) / p.BG;
    const int64_t max_ntb = (L + 63) / 64;
    if (ntb > max_ntb) ntb = max_ntb;
    if (ntb < 1) ntb = 1;
    while (ntb > 1 && p.BG * p.Nc * ntb > 131072) ntb = (ntb + 1) / 2;
    p.TB = (L + ntb - 1) / ntb;
    p.NTB = p.TB > 0 ? (L + p.TB - 1) / p.TB : 1;
    p.E = kSegRows / G;
    const int64_t n_entries = p.BG * L * topk;
    p.max_seg = p.BG * p.NcAll + p.BG * p.Nc + (n_entries + p.E - 1) / p.E;
    size_t off = kStatusBytes;
    p.lm_off = off;
    if (dhsa) off = align_up(off + sizeof(float) * (size_t)(p.BG * p.Nc * d), 256);
    p.coef_off = off;
    off = align_up(off + sizeof(float2) * (size_t)B * L * H * topk, 256);
    p.cnt_off = off;
    p.cnt_bytes = sizeof(int32_t) * (size_t)(p.BG * p.Nc * p.NTB > 0 ? p.BG * p.Nc * p.NTB : 1);
    off = align_up(off + p.cnt_bytes, 256);
    p.entries_off = off;
    off = align_up(off + sizeof(int32_t) * (size_t)(n_entries > 0 ? n_entries : 1), 256);
    p.segs_off = off;
    off = align_up(off + sizeof(int4) * (size_t)p.max_seg, 256);
    p.nseg_off = off;
    off = align_up(off + sizeof(int32_t), 256);
    p.cseg_off = off;
    off = align_up(off + 2 * sizeof(int32_t) * (size_t)(p.BG * p.NcAll), 256);
    p.part_off = off;
    off = align_up(off + sizeof(float) * 129 * (size_t)d * (size_t)p.max_seg, 256);
    p.dw_off = p.dqp_off = off;
    if (tc) {                // dw per (row, slot) and the dQ partial rows, own chunk last
        p.dw_off = off;
        off = align_up(off + sizeof(float) * (size_t)B * L * H * (topk + 1), 256);
        p.dqp_off = off;
        off = align_up(off + sizeof(__half) * (size_t)B * L * H * (topk + 1) * d, 256);
    }
    p.total = off;
    return p;
}

template <typename T, int D>
static cudaError_t launch_backward_t(const BwdArgs &a, const BwdLayout &p, cudaStream_t st) {
    char *ws = (char *)a.ws;
    const int G = a.H / a.Hkv;
    float2 *coef = (float2 *)(ws + p.coef_off);
    int32_t *cnt = (int32_t *)(ws + p.cnt_off);
    int32_t *entries = (int32_t *)(ws + p.entries_off);
    int4 *segs = (int4 *)(ws + p.segs_off);
    int32_t *nseg = (int32_t *)(ws + p.nseg_off);
    int32_t *cseg_beg = (int32_t *)(ws + p.cseg_off);
    int32_t *cseg_n = cseg_beg + p.BG * p.NcAll;
    float *part = (float *)(ws + p.part_off);
    unsigned *status = (unsigned *)ws;
    constexpr int VEC = Vec16<T>::N;

    // 1. dQ and the per-slot coefficients (CUDA cores), or the fusion weights
    //    alone (tensor-core path: dQ comes from the key pass)
    if (p.tc) {
        cudaError_t e = launch_backward_tc(a.Q, a.K, a.V, a.dO, a.lm, a.lm_bf16 != 0, a.idx, a.B,
                                           a.H, a.Hkv, a.L, a.S, p.Nc, p.NcAll, a.topk,
                                           a.own_chunk, a.scale, coef, nullptr, nullptr, nullptr,
                                           nullptr, nullptr, nullptr, 0, status, a.dQ, 0, st);
        if (e != cudaSuccess) return e;
    } else {
        const size_t smem = sizeof(float) * 2 * G * D + 2 * sizeof(T) * 64 * (D + VEC);
        auto kern = bwd_row_kernel<T, D>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<dim3((unsigned)a.L, (unsigned)a.Hkv, (unsigned)a.B), 32 * G, smem, st>>>(
            (const T *)a.Q, (const T *)a.K, (const T *)a.V, a.lm, a.lm_bf16, a.idx, (const T *)a.dO,
            a.H, a.Hkv, a.L, a.S, p.Nc, a.topk, a.own_chunk, a.scale, coef, a.dQ, status);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    // 2. stable per-chunk entry lists and the segments
    const size_t hsmem = sizeof(int32_t) * (size_t)p.Nc;
    const int use_smem = hsmem <= 160 * 1024 ? 1 : 0;
    if (p.Nc > 0) {
        cudaError_t e = cudaMemsetAsync(cnt, 0, p.cnt_bytes, st);
        if (e != cudaSuccess) return e;
        if (use_smem) {
            if ((e = cudaFuncSetAttribute(bwd_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)hsmem)) != cudaSuccess ||
                (e = cudaFuncSetAttribute(bwd_scatter_kernel,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, (int)hsmem)) !=
                    cudaSuccess)
                return e;
        }
        bwd_hist_kernel<<<dim3((unsigned)p.NTB, (unsigned)p.BG), 256, use_smem ? hsmem : 0, st>>>(
            a.idx, a.Hkv, a.L, a.S, p.Nc, a.topk, p.TB, p.NTB, use_smem, cnt);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    bwd_scan_kernel<<<1, kScanThreads2, 0, st>>>(cnt, p.BG, p.Nc, p.NcAll, p.NTB, a.own_chunk,
                                                 (int)p.E, segs, nseg, cseg_beg, cseg_n);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (p.Nc > 0) {
        bwd_scatter_kernel<<<dim3((unsigned)p.NTB, (unsigned)p.BG), 32, use_smem ? hsmem : 0, st>>>(
            a.idx, a.Hkv, a.L, a.S, p.Nc, a.topk, p.TB, p.NTB, use_smem, cnt, entries);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    // 3. per-segment dK / dV / dl partials
    if (p.tc) {
        e = launch_backward_tc(a.Q, a.K, a.V, a.dO, a.lm, a.lm_bf16 != 0, a.idx, a.B, a.H, a.Hkv,
                               a.L, a.S, p.Nc, p.NcAll, a.topk, a.own_chunk, a.scale, coef,
                               (float *)(ws + p.dw_off), (__half *)(ws + p.dqp_off), segs, nseg,
                               entries, part, p.max_seg, status, a.dQ, 1, st);
        if (e != cudaSuccess) return e;
    } else {
        const size_t smem =
            sizeof(float) * (2 * 64 * (D + kKeyLanes) + 2 * 8 * D + 3 * (kKeyThreads / 32) * 8);
        auto kern = bwd_key_kernel<T, D>;
        if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)smem)) != cudaSuccess)
            return e;
        kern<<<(unsigned)p.max_seg, kKeyThreads, smem, st>>>(
            (const T *)a.Q, (const T *)a.K, (const T *)a.V, (const T *)a.dO, coef, entries, segs,
            nseg, a.H, a.Hkv, a.L, a.S, p.NcAll, a.topk, a.scale, part);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    // 4. ordered reduction into dK, dV, dlm
    bwd_reduce_kernel<D><<<dim3((unsigned)(p.BG * p.NcAll), kReduceSlices), 256, 0, st>>>(
        part, cseg_beg, cseg_n, a.L, a.S, p.Nc, p.NcAll, a.dhsa, a.dK, a.dV, a.dlm);
    return cudaGetLastError();
}

cudaError_t launch_backward(const BwdArgs &a, const BwdLayout &p, cudaStream_t st) {
    if (a.bf16)
        return a.d == 128 ? launch_backward_t<__nv_bfloat16, 128>(a, p, st)
                          : launch_backward_t<__nv_bfloat16, 64>(a, p, st);
    return a.d == 128 ? launch_backward_t<float, 128>(a, p, st)
                      : launch_backward_t<float, 64>(a, p, st);
}

}  // namespace hsa
