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
// The landmark scan is the HBM stream; the K/V cache is read only for the K
// selected chunks.
//
// decode_scan_kernel: grid = splits x (B*Hkv), sized to one wave.  Each block
// owns a contiguous range of landmark rows.  A producer warp streams the range
// through a 4-stage shared-memory ring with 16 KB bulk async copies (full /
// empty mbarriers, so consumers never wait on a block-wide barrier); eight
// consumer warps score the rows: a quarter-warp holds one row, its dot product
// with the scaled qbar uses packed fp32 FMAs and three xor-shuffles.  A float
// threshold filters rows; only the rare candidates become 64-bit (score,
// ~index) keys in a warp-distributed top-K.  Blocks publish their K best keys
// and take a ticket; the last block of each (b, g) merges all candidates with
// warp-parallel selection, writes the selection and resets the ticket.  No
// block waits for another.  (Prefetching the selected K/V chunks into L2 from
// that block was tried: it lengthened the scan's tail by more than it saved
// the attend kernel.)
//
// decode_attend_kernel (launched as a programmatic dependent of the scan, so
// its launch and its query loads overlap the scan's tail): one cluster of
// min(K, 8) blocks per (b, g); see the kernel's comment.
//
// Context-parallel decode (a cache cut into contiguous chunk ranges, one per
// GPU) runs the same two kernels on each shard with a DecodeShard: the scan
// keys carry global chunk indices and its merge also writes the shard's top-K
// (score, index) candidates; after the candidates of all shards are gathered,
// decode_cp_merge_kernel takes the global top-K in the same total order; the
// attend kernel then folds only the selected chunks the shard holds and writes
// its per-head fusion state (m, Z, acc) instead of O; after the states are
// gathered, decode_cp_combine_kernel combines them in shard order.  A global
// top-K chunk is within its own shard's top K, so the result equals the
// single-GPU decode.
#include <cooperative_groups.h>

#include "common.cuh"
#include "tc.cuh"

namespace cg = cooperative_groups;

namespace hsa {

constexpr int kScanWarps = 8;                  // consumer warps
constexpr int kScanThreads = (kScanWarps + 1) * 32;   // + one producer warp
constexpr int kScanStages = 4;
constexpr int kStageBytes = 16384;
constexpr int kScanBlocksPerSm = 3;            // 64 KB ring + ~3 KB per block
constexpr long long kScanWait = 4000000000LL;  // SM cycles (about 2 s)

// Top-K of `nlists` (<= 8 * 32 / KP) sorted lists of KP keys held in shared
// memory (list l = lists[l][0 .. KP-1]); executed by one warp, lane k < KP
// returns the k-th best.
__device__ __forceinline__ uint64_t merge_smem_lists(const uint64_t (*lists)[32], int nlists,
                                                     int KP) {
    const int lane = threadIdx.x & 31;
    const int per = 32 / KP, li = lane / KP, e = lane % KP;
    const int nr = (nlists + per - 1) / per;
    uint64_t x[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const int l = r * per + li;
        x[r] = (r < nr && l < nlists) ? lists[l][e] : 0ull;
    }
    return merge_segments(merge_regs8(x, nr, KP), KP);
}

// Grid: splits * B*Hkv blocks, 1-D, interleaved over (b, g) so that the blocks
// of every (b, g) spread over all SMs.  Work is handed out in units of one
// ring stage (ROWS landmark rows) from a per-(b, g) counter, so that blocks on
// SMs that stream faster take more units.
template <typename T, typename TL, int D>
__global__ void __launch_bounds__(kScanThreads)
decode_scan_kernel(const T *__restrict__ q, const TL *__restrict__ lm, int H, int Hkv, int64_t Nc,
                   int topk, float scale, int splits, DecodeScratch ws, int32_t *__restrict__ idx_out,
                   DecodeShard sh) {
    constexpr int ROW_BYTES = D * (int)sizeof(TL);
    constexpr int ROWS = kStageBytes / ROW_BYTES;           // landmark rows per stage (one unit)
    constexpr int VEC = Vec16<TL>::N;                        // elements per 16-byte vector
    constexpr int LPR = 8;                                   // lanes per row (one quarter-warp)
    constexpr int VPL = D / VEC / LPR;                       // 16-byte vectors per lane and row
    constexpr int ITER = ROWS / (kScanWarps * 4);            // warp steps (4 rows each) per stage
    static_assert(ROWS % (kScanWarps * 4) == 0, "stage must split evenly over warps");
    static_assert(VPL >= 1, "row narrower than a quarter-warp");

    extern __shared__ __align__(128) uint8_t ring[];         // [kScanStages][kStageBytes]
    __shared__ uint64_t full[kScanStages], empty[kScanStages];
    __shared__ int64_t unit_of[kScanStages];                 // -1: no more units
    __shared__ float qbar_s[D];
    __shared__ uint64_t lists[kScanWarps][32];
    __shared__ int is_last, s_abort;

    const int64_t pairs = (int64_t)gridDim.x / splits;
    const int64_t bg = blockIdx.x % pairs;
    const int split = (int)(blockIdx.x / pairs);
    const int64_t b = bg / Hkv;
    const int g = (int)(bg % Hkv);
    const int G = H / Hkv;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const TL *lm_bg = lm + bg * Nc * D;
    const int KP = pow2_at_least(topk);
    grid_dep_wait();            // inputs and workspace may come from the previous kernel
    // chunks this sequence sees: all Nc, or its first lens[b] / S (ragged batch;
    // a length outside 0 .. Nc*S is flagged and clamped)
    int64_t nvis = Nc;
    if (sh.lens) {
        const int64_t len = sh.lens[b];
        if ((len < 0 || len > Nc * sh.S) && split == 0 && g == 0 && tid == 0)
            atomicOr(ws.status, kFlagBadBounds);
        nvis = len < 0 ? 0 : len > Nc * sh.S ? Nc : len / sh.S;
    }
    const int64_t nunits = (nvis + ROWS - 1) / ROWS;

    if (tid == 0) {
        for (int i = 0; i < kScanStages; ++i) {
            tc::mbar_init(&full[i], 1);
            tc::mbar_init(&empty[i], kScanWarps);
        }
        s_abort = 0;
        tc::fence_barrier_init();
    }
    __syncthreads();

    WarpTopK tk;
    tk.init(topk);
    uint64_t thr = 0ull;
    if (warp == kScanWarps) {
        // producer: one lane claims units (one claim ahead, so the atomic's
        // latency overlaps the wait for a free slot) and keeps kScanStages
        // bulk copies in flight; a unit of -1 tells the consumers to stop
        if (lane == 0) {
            int64_t u_next = (int64_t)atomicAdd(ws.next_unit + bg, 1u);
            int64_t st = 0;
            for (;; ++st) {
                const int slot = (int)(st % kScanStages);
                if (st >= kScanStages &&
                    !tc::mbar_wait(&empty[slot], (uint32_t)(((st / kScanStages) - 1) & 1),
                                   kScanWait)) {
                    s_abort = 1;
                    break;
                }
                const int64_t u = u_next;
                if (u >= nunits) {
                    unit_of[slot] = -1;
                    tc::mbar_arrive(&full[slot]);
                    ++st;
                    break;
                }
                u_next = (int64_t)atomicAdd(ws.next_unit + bg, 1u);
                const int64_t row0 = u * ROWS;
                const int64_t left = nvis - row0;
                const uint32_t bytes = (uint32_t)((left < ROWS ? left : ROWS) * ROW_BYTES);
                unit_of[slot] = u;
                tc::mbar_expect_tx(&full[slot], bytes);
                tc::bulk_load(ring + slot * kStageBytes, lm_bg + row0 * D, bytes, &full[slot]);
            }
            // the copies still in flight land before the block can exit
            for (int64_t j = st > kScanStages ? st - kScanStages : 0; j < st; ++j)
                tc::mbar_wait(&full[j % kScanStages], (uint32_t)((j / kScanStages) & 1), kScanWait);
        }
    } else {
        // qbar (consumer warps only, while the first copies are in flight)
        for (int j = tid; j < D; j += kScanWarps * 32) {
            const T *qp = q + (b * H + (int64_t)g * G) * D + j;
            float a = 0.f;
#pragma unroll 4
            for (int h = 0; h < G; ++h) a += to_f32(qp[(int64_t)h * D]);
            qbar_s[j] = a / (float)G;
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kScanWarps * 32) : "memory");
        // the 8 lanes of quarter-warp `sub` share one row; lane c holds the
        // 16-byte vectors c, c + 8, ... of it and the matching scaled qbar pairs
        const int c = lane & 7, sub = lane >> 3;
        constexpr int PAIRS = Dot16<TL>::PAIRS;
        uint64_t q2[VPL][PAIRS];
#pragma unroll
        for (int j = 0; j < VPL; ++j)
#pragma unroll
            for (int e = 0; e < PAIRS; ++e) {
                const float *qp = qbar_s + (c + LPR * j) * VEC + 2 * e;
                q2[j][e] = pack_f2(scale * qp[0], scale * qp[1]);
            }
        float tf = -INFINITY;          // score of the K-th best key so far
        for (int64_t st = 0;; ++st) {
            const int slot = (int)(st % kScanStages);
            if (!tc::mbar_wait(&full[slot], (uint32_t)((st / kScanStages) & 1), kScanWait)) {
                s_abort = 1;
                break;
            }
            const int64_t unit = unit_of[slot];
            if (unit < 0) break;
            const int64_t row0 = unit * ROWS;
            const int rows_here = (int)(nvis - row0 < ROWS ? nvis - row0 : ROWS);
            const uint8_t *stage = ring + slot * kStageBytes;
#pragma unroll
            for (int it = 0; it < ITER; ++it) {
                const int rr = (it * kScanWarps + warp) * 4 + sub;
                const uint8_t *row = stage + rr * ROW_BYTES;
                uint64_t acc = 0ull;
#pragma unroll
                for (int j = 0; j < VPL; ++j)
                    acc = Dot16<TL>::fma(*reinterpret_cast<const uint4 *>(row + (c + LPR * j) * 16),
                                         q2[j], acc);
                float a = sum_f2(acc);
                a += __shfl_xor_sync(0xffffffffu, a, 4);
                a += __shfl_xor_sync(0xffffffffu, a, 2);
                a += __shfl_xor_sync(0xffffffffu, a, 1);
                // cheap float filter; ties and the exact order are settled on the keys
                unsigned m = __ballot_sync(0xffffffffu, a >= tf && rr < rows_here) & 0x01010101u;
                if (m) {
                    const uint64_t key = make_key(a, sh.c0 + row0 + rr);
                    while (m) {
                        const int s = __ffs(m) - 1;
                        m &= m - 1;
                        const uint64_t x = __shfl_sync(0xffffffffu, key, s);
                        if (x > thr) {
                            tk.insert(x);
                            thr = tk.threshold();
                        }
                    }
                    tf = key_score(thr);
                }
            }
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&empty[slot]);     // this warp is done with the slot
        }
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // block merge of the warp lists
    if (warp < kScanWarps) lists[warp][lane] = tk.v;
    __syncthreads();
    if (warp == 0) {
        const uint64_t best = merge_smem_lists(lists, kScanWarps, KP);
        if (lane < topk) ws.cand[(bg * splits + split) * topk + lane] = best;
        __threadfence();                      // the candidates before the ticket
    }
    if (s_abort && tid == 0) atomicOr(ws.status, kFlagTimeout);

    // last block of this (b, g) merges the candidates of every block
    __syncthreads();
    if (tid == 0) is_last = (atomicAdd(&ws.tickets[bg], 1u) == (unsigned)(splits - 1));
    __syncthreads();
    if (!is_last || warp >= kScanWarps) return;
    __threadfence();
    // each consumer warp merges groups of 32/KP block lists (warp w: groups
    // w, w + 8, ...), eight groups per load batch, merged as a tree
    const uint64_t *cb = ws.cand + bg * splits * topk;
    const int per = 32 / KP, li = lane / KP, e = lane % KP;
    const int64_t ngroups = (splits + per - 1) / per;
    uint64_t acc = 0ull;
    for (int64_t g0 = warp; g0 < ngroups; g0 += 8 * kScanWarps) {
        uint64_t x[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int64_t gi = g0 + (int64_t)u * kScanWarps;
            const int64_t l = gi * per + li;
            x[u] = (gi < ngroups && l < splits && e < topk)
                       ? (uint64_t)__ldcg(reinterpret_cast<const unsigned long long *>(cb + l * topk + e))
                       : 0ull;
        }
        acc = merge_lists(acc, merge_regs8(x, 8, KP), KP);
    }
    lists[warp][lane] = merge_segments(acc, KP);
    asm volatile("bar.sync 1, %0;" ::"n"(kScanWarps * 32) : "memory");
    if (warp == 0) {
        const uint64_t best = merge_smem_lists(lists, kScanWarps, KP);
        if (lane < topk) {
            const int32_t i = key_index(best);
            ws.sel[bg * topk + lane] = i;
            if (idx_out) idx_out[bg * topk + lane] = i;
            if (sh.cand_idx) {                // the shard's candidates for the exchange
                sh.cand_idx[bg * topk + lane] = i;
                sh.cand_score[bg * topk + lane] = key_score(best);
            }
        }
        if (lane == 0) {                      // ready for the next call
            ws.tickets[bg] = 0u;
            ws.next_unit[bg] = 0u;
        }
    }
}

// decode_attend_kernel: one thread-block cluster of C = min(K, 8) blocks per
// (b, g); block c of the cluster takes the slots k = c, c + C, ...  For every
// slot it stages the chunk's K and V, and for each head h computes the fusion
// logit z = scale * q_h . l_k and the chunk output o (softmax inside the
// chunk).  Across its slots a block keeps per head the running maximum m,
// the sum Z of exp(z - m) and acc = sum of exp(z - m) * o, so that the
// fusion softmax over the K slots is exact once the C partial states are
// combined: O = sum_c exp(m_c - M) acc_c / sum_c exp(m_c - M) Z_c, M = max m_c.
// The blocks combine through distributed shared memory, each writing its
// share of O, in a fixed order (deterministic).
constexpr int kAttThreads = 256;
constexpr int kAttWarps = kAttThreads / 32;
constexpr int kAttMaxCluster = 8;

// R consecutive elements of a shared-memory row as fp32, one load instruction.
template <typename T, int R>
__device__ __forceinline__ void load_row_slice(const T *p, float (&v)[R]);
template <>
__device__ __forceinline__ void load_row_slice<__nv_bfloat16, 4>(const __nv_bfloat16 *p, float (&v)[4]) {
    const uint2 u = *reinterpret_cast<const uint2 *>(p);
    v[0] = __uint_as_float(u.x << 16); v[1] = __uint_as_float(u.x & 0xffff0000u);
    v[2] = __uint_as_float(u.y << 16); v[3] = __uint_as_float(u.y & 0xffff0000u);
}
template <>
__device__ __forceinline__ void load_row_slice<__nv_bfloat16, 2>(const __nv_bfloat16 *p, float (&v)[2]) {
    const uint32_t u = *reinterpret_cast<const uint32_t *>(p);
    v[0] = __uint_as_float(u << 16); v[1] = __uint_as_float(u & 0xffff0000u);
}
template <>
__device__ __forceinline__ void load_row_slice<float, 4>(const float *p, float (&v)[4]) {
    const float4 u = *reinterpret_cast<const float4 *>(p);
    v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
}
template <>
__device__ __forceinline__ void load_row_slice<float, 2>(const float *p, float (&v)[2]) {
    const float2 u = *reinterpret_cast<const float2 *>(p);
    v[0] = u.x; v[1] = u.y;
}

template <typename T, int D>
struct AttSmem {
    static constexpr int VT = Vec16<T>::N;
    static constexpr int RS = D + VT;                       // padded K/V row (elements)
    // fp32 q [G][D], acc [G][D], m [16], Z [16], lrow [D], p [warps][64], then the
    // K and V tiles; every region starts on a 16-byte boundary (G <= 16, D % 64 == 0)
    static size_t bytes(int G) {
        return sizeof(float) * (2 * (size_t)G * D + 2 * 16 + D + kAttWarps * 64) +
               2 * sizeof(T) * 64 * RS;
    }
};

template <typename T, typename TL, int D>
__global__ void __launch_bounds__(kAttThreads)
decode_attend_kernel(const T *__restrict__ q, const TL *__restrict__ lm, const T *__restrict__ Kc,
                     const T *__restrict__ Vc, int H, int Hkv, int64_t Lc, int S, int topk,
                     float scale, const int32_t *__restrict__ sel, T *__restrict__ O,
                     DecodeShard sh) {
    constexpr int VT = AttSmem<T, D>::VT;
    constexpr int RS = AttSmem<T, D>::RS;
    constexpr int R = D / 32;
    constexpr int VPR = D / VT;                              // 16-byte vectors per K/V row
    constexpr int NV = 64 * VPR / kAttThreads;               // vectors per thread, K and V each
    constexpr int LV = D * (int)sizeof(TL) / 16;             // 16-byte vectors per landmark row
    static_assert(NV >= 1 && (64 * VPR) % kAttThreads == 0, "K/V tile must split over threads");
    cg::cluster_group cluster = cg::this_cluster();
    extern __shared__ float4 dyn4[];
    const int C = (int)cluster.num_blocks();
    const int crank = (int)cluster.block_rank();
    const int64_t bg = blockIdx.y;
    const int64_t b = bg / Hkv;
    const int g = (int)(bg % Hkv);
    const int G = H / Hkv;
    const int64_t Nc = Lc / S;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    float *qs = reinterpret_cast<float *>(dyn4);                  // [G][D]
    float *acc_s = qs + G * D;                                    // [G][D]
    float *m_s = acc_s + G * D;                                   // [G], 16 reserved
    float *z_s = m_s + 16;                                        // [G], 16 reserved
    float *lrow = z_s + 16;                                       // [D]
    float *ps = lrow + D;                                         // [warps][64]
    T *ks = reinterpret_cast<T *>(ps + kAttWarps * 64);           // [64][RS]
    T *vs = ks + 64 * RS;

    // the queries are an input: load them before waiting for the scan
    {
        const T *qg = q + (b * H + g * G) * (int64_t)D;
        for (int e = tid; e < G * VPR; e += kAttThreads) {
            float f[VT];
            Vec16<T>::unpack(*reinterpret_cast<const uint4 *>(qg + e * VT), f);
#pragma unroll
            for (int u = 0; u < VT; ++u) qs[e * VT + u] = f[u];
        }
        for (int e = tid; e < G * D; e += kAttThreads) acc_s[e] = 0.f;
        for (int e = tid; e < G; e += kAttThreads) {
            m_s[e] = -INFINITY;
            z_s[e] = 0.f;
        }
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");   // the selection is written by the scan

    for (int k = crank; k < topk; k += C) {
        const int32_t cg_ = sel[bg * topk + k];
        if (cg_ < 0) break;                    // padding only at the end of the selection
        const int64_t ci = (int64_t)cg_ - sh.c0;        // index within this cache (shard)
        if (ci < 0 || ci >= Nc) continue;      // another shard's chunk (block-uniform)
        __syncthreads();                       // previous slot's tiles are no longer read
        {
            const int64_t first = (int64_t)ci * S;
            const T *Kb = Kc + (bg * Lc + first) * D;
            const T *Vb = Vc + (bg * Lc + first) * D;
            uint4 kr[NV], vr[NV];
#pragma unroll
            for (int u = 0; u < NV; ++u) {
                const int e = tid + u * kAttThreads;
                kr[u] = ld_stream16(Kb + (int64_t)e * VT);
                vr[u] = ld_stream16(Vb + (int64_t)e * VT);
            }
            uint4 lr = make_uint4(0, 0, 0, 0);
            const TL *lp = lm + (bg * Nc + ci) * D;
            if (tid < LV)
                lr = *reinterpret_cast<const uint4 *>(reinterpret_cast<const uint8_t *>(lp) + tid * 16);
#pragma unroll
            for (int u = 0; u < NV; ++u) {
                const int e = tid + u * kAttThreads;
                const int r = e / VPR, c = (e % VPR) * VT;
                *reinterpret_cast<uint4 *>(ks + r * RS + c) = kr[u];
                *reinterpret_cast<uint4 *>(vs + r * RS + c) = vr[u];
            }
            if (tid < LV) {
                constexpr int LE = Vec16<TL>::N;
                float f[LE];
                Vec16<TL>::unpack(lr, f);
#pragma unroll
                for (int u = 0; u < LE; ++u) lrow[tid * LE + u] = f[u];
            }
        }
        __syncthreads();
        for (int h = warp; h < G; h += kAttWarps) {
            const float *qh = qs + h * D;
            // fusion logit scale * q_h . l_ci
            float a = 0.f;
#pragma unroll
            for (int r = 0; r < R; ++r) a = fmaf(qh[lane + 32 * r], lrow[lane + 32 * r], a);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
            const float zl = scale * a;
            // in-chunk scores: lane takes keys lane and lane + 32, two partial sums each
            float sc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
#pragma unroll 2
            for (int c = 0; c < D / 2; c += VT) {
#pragma unroll
                for (int u = 0; u < 2; ++u)
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        const int cc = c + hf * (D / 2);
                        float f[VT];
                        Vec16<T>::unpack(
                            *reinterpret_cast<const uint4 *>(ks + (lane + 32 * u) * RS + cc), f);
#pragma unroll
                        for (int e = 0; e < VT; ++e) sc[u][hf] = fmaf(qh[cc + e], f[e], sc[u][hf]);
                    }
            }
            const float l0 = scale * (sc[0][0] + sc[0][1]), l1 = scale * (sc[1][0] + sc[1][1]);
            float mx = fmaxf(l0, l1);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            const float p0 = expf(l0 - mx), p1 = expf(l1 - mx);
            float den = p0 + p1;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
            float *pw = ps + warp * 64;
            pw[lane] = p0;
            pw[lane + 32] = p1;
            __syncwarp();
            // P.V: lane owns the R consecutive elements R*lane .. R*lane + R - 1
            float o_r[R];
#pragma unroll
            for (int r = 0; r < R; ++r) o_r[r] = 0.f;
#pragma unroll 8
            for (int j = 0; j < 64; ++j) {
                const float pj = pw[j];
                float v[R];
                load_row_slice<T, R>(vs + j * RS + R * lane, v);
#pragma unroll
                for (int r = 0; r < R; ++r) o_r[r] = fmaf(pj, v[r], o_r[r]);
            }
            __syncwarp();
            // fold (zl, o / den) into this block's running fusion state of head h
            const float m_old = m_s[h];
            const float m_new = fmaxf(m_old, zl);
            const float c_old = expf(m_old - m_new);          // 0 while the state is empty
            const float c_new = expf(zl - m_new);
            const float f = c_new / den;
            float *ah = acc_s + h * D + R * lane;
#pragma unroll
            for (int r = 0; r < R; ++r) ah[r] = ah[r] * c_old + o_r[r] * f;
            __syncwarp();
            if (lane == 0) {
                z_s[h] = z_s[h] * c_old + c_new;
                m_s[h] = m_new;
            }
            __syncwarp();
        }
    }

    // combine the C block states of this (b, g); block c writes heads c, c + C, ...
    // (all remote loads of a head are issued before any is used)
    cluster.sync();
    for (int h = crank + C * warp; h < G; h += C * kAttWarps) {
        float mr[kAttMaxCluster], zr[kAttMaxCluster];
#pragma unroll
        for (int r = 0; r < kAttMaxCluster; ++r) {
            mr[r] = r < C ? cluster.map_shared_rank(m_s, r)[h] : -INFINITY;
            zr[r] = r < C ? cluster.map_shared_rank(z_s, r)[h] : 0.f;
        }
        float ar[kAttMaxCluster][R];
#pragma unroll
        for (int r = 0; r < kAttMaxCluster; ++r)
#pragma unroll
            for (int i = 0; i < R; ++i)
                ar[r][i] = r < C ? cluster.map_shared_rank(acc_s, r)[h * D + R * lane + i] : 0.f;
        float M = -INFINITY;
#pragma unroll
        for (int r = 0; r < kAttMaxCluster; ++r) M = fmaxf(M, mr[r]);
        float Z = 0.f;
        float o_r[R];
#pragma unroll
        for (int i = 0; i < R; ++i) o_r[i] = 0.f;
#pragma unroll
        for (int r = 0; r < kAttMaxCluster; ++r) {
            const float cr = mr[r] > -INFINITY ? expf(mr[r] - M) : 0.f;   // 0: block had no slot
            Z = fmaf(zr[r], cr, Z);
#pragma unroll
            for (int i = 0; i < R; ++i) o_r[i] = fmaf(ar[r][i], cr, o_r[i]);
        }
        const int64_t bh = b * H + g * G + h;
        if (sh.acc) {                          // this shard's fusion state instead of O
            float *ap = sh.acc + bh * D + R * lane;
#pragma unroll
            for (int i = 0; i < R; ++i) ap[i] = o_r[i];
            if (lane == 0) {
                sh.m[bh] = M;
                sh.Z[bh] = Z;
            }
            continue;
        }
        const float inv = Z > 0.f ? 1.f / Z : 0.f;
        T *op = O + bh * (int64_t)D + R * lane;
#pragma unroll
        for (int i = 0; i < R; ++i) op[i] = from_f32<T>(o_r[i] * inv);
    }
    cluster.sync();          // no block leaves while another still reads its state
}

// Blocks per (b, g): as many as fit in one wave (kScanBlocksPerSm per SM),
// at least one, and no more than one per 256 landmark rows.
int decode_splits(int B, int Hkv, int64_t Nc, int num_sms) {
    const int64_t pairs = (int64_t)B * Hkv;
    int64_t s = (int64_t)kScanBlocksPerSm * num_sms / pairs;
    const int64_t max_s = (Nc + 255) / 256;
    if (s > max_s) s = max_s;
    if (s < 1) s = 1;
    return (int)s;
}

// ---------------------------------------------------------------- context parallel
// Global top-K over R shards' candidates (gathered [R][B*Hkv][topk] scores and
// global indices, -1 for none), one warp per (b, g): every candidate above the
// current K-th key enters a warp-distributed sorted list; keys order (score,
// then lower index) totally, so the visiting order does not matter.
__global__ void __launch_bounds__(32)
decode_cp_merge_kernel(const float *__restrict__ score, const int32_t *__restrict__ cidx, int R,
                       int64_t pairs, int topk, int32_t *__restrict__ idx) {
    const int64_t bg = blockIdx.x;
    const int lane = threadIdx.x;
    WarpTopK tk;
    tk.init(topk);
    uint64_t thr = 0ull;
    const int64_t n = (int64_t)R * topk;
    for (int64_t i0 = 0; i0 < n; i0 += 32) {
        const int64_t i = i0 + lane;
        uint64_t key = 0ull;
        if (i < n) {
            const int64_t r = i / topk, k = i % topk;
            const int64_t at = (r * pairs + bg) * topk + k;
            const int32_t ci = cidx[at];
            if (ci >= 0) key = make_key(score[at], ci);
        }
        unsigned m = __ballot_sync(0xffffffffu, key > thr);
        while (m) {
            const int s = __ffs(m) - 1;
            m &= m - 1;
            const uint64_t x = __shfl_sync(0xffffffffu, key, s);
            if (x > thr) {
                tk.insert(x);
                thr = tk.threshold();
            }
        }
    }
    if (lane < topk) idx[bg * topk + lane] = key_index(tk.v);
}

// O from R shards' fusion states (gathered [R][B*H] m, Z and [R][B*H][D] acc),
// combined in shard order: O = sum_r e^{m_r - M} acc_r / sum_r e^{m_r - M} Z_r,
// M = max_r m_r; a shard that held no selected chunk has m = -inf.  One warp
// per (b, h).
template <typename T>
__global__ void __launch_bounds__(256)
decode_cp_combine_kernel(const float *__restrict__ m, const float *__restrict__ Z,
                         const float *__restrict__ acc, int R, int64_t rows, int D,
                         T *__restrict__ O) {
    const int64_t bh = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (bh >= rows) return;
    float M = -INFINITY;
    for (int r = 0; r < R; ++r) M = fmaxf(M, m[(int64_t)r * rows + bh]);
    float z = 0.f;
    for (int r = 0; r < R; ++r) {
        const float mr = m[(int64_t)r * rows + bh];
        z += mr > -INFINITY ? expf(mr - M) * Z[(int64_t)r * rows + bh] : 0.f;
    }
    const float inv = z > 0.f ? 1.f / z : 0.f;
    for (int c = lane; c < D; c += 32) {
        float a = 0.f;
        for (int r = 0; r < R; ++r) {
            const float mr = m[(int64_t)r * rows + bh];
            if (mr > -INFINITY) a = fmaf(expf(mr - M), acc[((int64_t)r * rows + bh) * D + c], a);
        }
        O[bh * D + c] = from_f32<T>(a * inv);
    }
}

// What a decode launch runs: both kernels (a whole cache), the scan only
// (a shard's candidates) or the attend kernel only (a shard's state).
enum DecodeStages { kDecodeBoth = 0, kDecodeScanOnly = 1, kDecodeAttendOnly = 2 };

template <typename T, typename TL, int D>
static cudaError_t launch_decode_t(const void *q, const void *lm, const void *Kc, const void *Vc,
                                   int B, int H, int Hkv, int64_t Lc, int S, int topk,
                                   float scale, int splits, const DecodeScratch &ws, void *O,
                                   int32_t *idx_out, const DecodeShard &sh, int stages,
                                   const int32_t *sel, cudaStream_t st) {
    const int64_t Nc = Lc / S;
    const unsigned grid = (unsigned)((int64_t)splits * B * Hkv);
    cudaError_t e;
    if (stages != kDecodeAttendOnly) {
        auto scan = decode_scan_kernel<T, TL, D>;
        e = cudaFuncSetAttribute(scan, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kScanStages * kStageBytes);
        if (e != cudaSuccess) return e;
        // a programmatic dependent of whatever precedes it on the stream (it waits
        // for that before reading anything), so its launch overlaps the tail
        e = launch_pdl(scan, dim3(grid), dim3(kScanThreads), (size_t)(kScanStages * kStageBytes),
                       st, (const T *)q, (const TL *)lm, H, Hkv, Nc, topk, scale, splits, ws,
                       idx_out, sh);
        if (e != cudaSuccess || stages == kDecodeScanOnly) return e;
    }

    const size_t smem = AttSmem<T, D>::bytes(H / Hkv);
    auto kern = decode_attend_kernel<T, TL, D>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // clusters of up to 8 blocks (one slot each) while 8 blocks per (b, g)
    // fit in about two waves; with more (b, g) pairs, 4 blocks of two slots
    // each place more easily and run faster (measured: batched decode
    // 69 -> 64.5 us; a single long sequence prefers 8)
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int cmax = (int64_t)B * Hkv * kAttMaxCluster <= 2 * (int64_t)sms ? kAttMaxCluster : 4;
    const int C = topk < cmax ? topk : cmax;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)C, (unsigned)(B * Hkv));
    cfg.blockDim = dim3(kAttThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, (const T *)q, (const TL *)lm, (const T *)Kc,
                              (const T *)Vc, H, Hkv, Lc, S, topk, scale,
                              sel ? sel : (const int32_t *)ws.sel, (T *)O, sh);
}

cudaError_t launch_decode(const void *q, const void *Kc, const void *Vc, bool bf16,
                          const void *lm, bool lm_bf16, int B, int H, int Hkv, int64_t Lc, int d,
                          int S, int topk, float scale, int splits, const DecodeScratch &ws,
                          void *O, int32_t *idx_out, const DecodeShard &sh, int stages,
                          const int32_t *sel, cudaStream_t st) {
#define HSA_DEC(T, TL, DD) \
    return launch_decode_t<T, TL, DD>(q, lm, Kc, Vc, B, H, Hkv, Lc, S, topk, scale, splits, ws, O, \
                                      idx_out, sh, stages, sel, st)
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

cudaError_t launch_decode_cp_merge(const float *score, const int32_t *cidx, int R, int B, int Hkv,
                                   int topk, int32_t *idx, cudaStream_t st) {
    const int64_t pairs = (int64_t)B * Hkv;
    decode_cp_merge_kernel<<<(unsigned)pairs, 32, 0, st>>>(score, cidx, R, pairs, topk, idx);
    return cudaGetLastError();
}

cudaError_t launch_decode_cp_combine(const float *m, const float *Z, const float *acc, int R,
                                     int B, int H, int d, bool bf16, void *O, cudaStream_t st) {
    const int64_t rows = (int64_t)B * H;
    const unsigned blocks = (unsigned)((rows + 7) / 8);
    if (bf16)
        decode_cp_combine_kernel<__nv_bfloat16><<<blocks, 256, 0, st>>>(m, Z, acc, R, rows, d,
                                                                       (__nv_bfloat16 *)O);
    else
        decode_cp_combine_kernel<float><<<blocks, 256, 0, st>>>(m, Z, acc, R, rows, d, (float *)O);
    return cudaGetLastError();
}

}  // namespace hsa
