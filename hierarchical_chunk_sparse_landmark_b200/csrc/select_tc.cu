// select_tc.cu -- prefill chunk selection with the group scores on the
// 5th-generation tensor cores.
//
// For each (b, t, g): qbar = mean of the G heads' queries, sbar_i = scale *
// qbar . l_i over the visible chunks i < floor(t/S), and the top-K chunks by
// (score desc, index asc).  (Per-token top-K retrieval over chunk landmarks:
// Understanding and Improving Length Generalization in Hierarchical Sparse
// Attention Models, "Methodology in Plain English".)
//
// Per (b, g) the scores are the dense product [L x d] . [d x Nc] (block-causal:
// only chunks before a token's own chunk count), so they run as tcgen05 MMA
// tiles: M = 128 tokens, N = 128 chunks, K = d, fp32 accumulate in TMEM.
// bf16 operands keep fp32 accuracy by splitting: qbar = q0 + q1 + q2 (three
// bf16 parts, exact for an fp32 value) against bf16 landmarks, or, for fp32
// landmarks l = l0 + l1, qbar = q0 + q1 and the products q0.l0 + q1.l0 + q0.l1
// (the q1.l1 term is below 2^-16 of the score and dropped).  The parts are
// chained as one accumulation per tile.
//
// select_tc_kernel: one block per (128-token block, b*Hkv + g), heavy blocks
// first.  All warps first build the qbar parts in shared memory (128-byte
// swizzled, K-major); then
//   warp 0      producer  (TMA of landmark tiles, two stages)
//   warp 1      MMA issuer (one score tile per landmark tile, two TMEM buffers)
//   warps 2-9   top-K     (thread = token = TMEM lane: causal mask, a sorted
//                          register list of (score, chunk) pairs, insertion
//                          only past the current K-th score; two groups of
//                          four warps over alternate 32-column blocks, lists
//                          merged at the end)
//   warps 10-11 L2 prefetch of the query rows of the block likely to start a
//               wave later, so that its qbar loads hit L2
// (the first two landmark tiles are requested before qbar is built, so their
// loads overlap it.)
// select_tc_half_kernel takes the case where every chunk fits one score tile
// (Nc <= 128): qbar built per 64-column block of d into one buffer, two blocks
// per SM (see the comment above it).
// Every wait is bounded; on expiry the block sets the status flag, lets its
// copies and MMAs land, frees its TMEM and exits.
#include <cuda.h>
#include <stdlib.h>
#include <string.h>

#include "common.cuh"
#include "tc.cuh"

namespace hsa {

template <int D, bool LM32>
struct SelCfg {
    static constexpr int M = 128;                 // tokens per block
    static constexpr int N = 128;                 // chunks per score tile (four stages of
                                                  // 64 chunks were tried: slower)
    static constexpr int KB = D / 64;             // 64-element blocks of d
    static constexpr int QP = LM32 ? 2 : 3;       // qbar parts
    static constexpr int LP = LM32 ? 2 : 1;       // landmark parts
    static constexpr int A_PART = M * D * 2;
    static constexpr int B_PART = N * D * 2;
    static constexpr int STAGES = 2;
    static constexpr int B_STAGE = LP * B_PART;
    static constexpr int BAR_OFF = QP * A_PART + STAGES * B_STAGE;
    static constexpr int STAGE_OFF = BAR_OFF + 256;      // top-K score rows [2 groups][32][128] fp32
    static constexpr int SMEM = 1024 + STAGE_OFF + 2 * 32 * 128 * 4;
    static_assert(STAGES * B_STAGE >= 32 * 128 * 8, "top-K lists must fit the landmark stages");
    static constexpr uint32_t TMEM_COLS = 2 * N;
};

constexpr int kSelTcThreads = 384;                  // 12 warps (6-11 only help build qbar)
constexpr long long kSelWait = 4000000000LL;        // SM cycles (about 2 s)

struct SelTcParams {
    const void *Q;                  // [B, L, H, D] bf16
    int32_t *idx;                   // [B, L, Hkv, topk]
    unsigned *status;
    int64_t L, Nc;
    int H, Hkv, S, topk;
    float scale;
    // one selection per R consecutive tokens (R divides S): selection row u
    // serves tokens u*R .. u*R+R-1; its group query is token u*R's
    // (pool_mean = 0) or the mean over the row's tokens (pool_mean = 1)
    int64_t Lsel;                   // selection rows, ceil(L / R)
    int R, pool_mean;
    Chunks ch;                      // chunks of S tokens or variable-length ones (R = 1)
};

// Number of (token, head) query rows summed into the group query of
// selection row u: the G heads of token u*R, or of every token of the row
// (pool_mean).  Eight consecutive pairs share a token (G is a multiple of 8
// on the tensor-core path).
__device__ __forceinline__ int qbar_pairs(const SelTcParams &p, int G, int64_t u) {
    if (!p.pool_mean) return G;
    const int64_t left = p.L - u * p.R;
    return G * (int)(left < p.R ? left : p.R);
}

__device__ __forceinline__ bool sel_wait(uint64_t *bar, uint32_t parity, volatile int *abort) {
    if (tc::mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!tc::mbar_try_wait(bar, parity)) {
        if (*abort || clock64() - t0 > kSelWait) {
            *abort = 1;
            return false;
        }
    }
    return true;
}

__device__ __forceinline__ uint32_t bf16_bits_rn(float x) {
    return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(x));
}

// A token's running top-K: scores s[0] >= s[1] >= ... (scaled group scores)
// and their chunk indices; empty slots hold (-inf, -1).  The order is score
// descending, then chunk index ascending (a total order: indices are distinct).
template <int KP>
struct TopList {
    float s[KP];
    int32_t i[KP];
    __device__ __forceinline__ void clear() {
#pragma unroll
        for (int k = 0; k < KP; ++k) {
            s[k] = -INFINITY;
            i[k] = -1;
        }
    }
    // above[k]: slot k ranks above the new entry and keeps what it holds;
    // the first other slot takes the new entry and every later one its upper
    // neighbour's.  The KP comparisons are independent of each other, so the
    // insertion is a few dependent steps, not a chain through the list; an
    // entry that ranks below every held one leaves the list as it is.
    __device__ __forceinline__ void place(const bool (&above)[KP], float xs, int32_t xi) {
#pragma unroll
        for (int k = KP - 1; k > 0; --k) {
            s[k] = above[k] ? s[k] : (above[k - 1] ? xs : s[k - 1]);
            i[k] = above[k] ? i[k] : (above[k - 1] ? xi : i[k - 1]);
        }
        s[0] = above[0] ? s[0] : xs;
        i[0] = above[0] ? i[0] : xi;
    }
    // Insert chunk xi whose index is above every held one (the columns of a
    // row arrive in index order): a held entry of equal score ranks first, so
    // a single float comparison per slot decides.
    __device__ __forceinline__ void insert_later(float xs, int32_t xi) {
        bool above[KP];
#pragma unroll
        for (int k = 0; k < KP; ++k) above[k] = s[k] >= xs;
        place(above, xs, xi);
    }
    // Insert an entry of any index (merging two lists).
    __device__ __forceinline__ void insert_any(float xs, int32_t xi) {
        bool above[KP];
#pragma unroll
        for (int k = 0; k < KP; ++k) above[k] = s[k] > xs || (s[k] == xs && (uint32_t)i[k] < (uint32_t)xi);
        place(above, xs, xi);
    }
};

// One 32-column block of a token's scores (chunks c0 .. c0+31, of which the
// first `lim` are visible) into its running top-K v.  The lane first marks
// its candidates -- unscaled scores at or above its current K-th score divided
// by the scale, a bound loosened by 1e-6 so that no column whose scaled score
// reaches it is missed; the exact test follows -- then takes them one per
// loop trip from its own 32-float row of `stage` (shared memory, column-major
// so the rows of a warp's lanes share no bank): the warp runs as many trips as
// its busiest lane needs, instead of the insertion at every column where any
// lane has a candidate.  Candidates are taken in column order, so each enters
// after every lower index.
// Sorts eight values into descending order (a 19-comparator network).
__device__ __forceinline__ void sort8_desc(float (&a)[8]) {
    constexpr int P[19][2] = {{0, 2}, {1, 3}, {4, 6}, {5, 7}, {0, 4}, {1, 5}, {2, 6},
                              {3, 7}, {0, 1}, {2, 3}, {4, 5}, {6, 7}, {2, 4}, {3, 5},
                              {1, 4}, {3, 6}, {1, 2}, {3, 4}, {5, 6}};
#pragma unroll
    for (int e = 0; e < 19; ++e) {
        const float hi = fmaxf(a[P[e][0]], a[P[e][1]]), lo = fminf(a[P[e][0]], a[P[e][1]]);
        a[P[e][0]] = hi;
        a[P[e][1]] = lo;
    }
}
// A lower bound on the 8th largest of the 64 scores x, y: the 8th largest of
// the 16 maxima of 4-column groups (eight distinct scores, each at or above
// it).  With both groups' maxima sorted, the 8 largest of the union are
// max(a[i], b[7-i]), so the bound is their minimum.
__device__ __forceinline__ float eighth_bound64(const float (&x)[32], const float (&y)[32]) {
    float a[8], b[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        a[q] = fmaxf(fmaxf(x[4 * q], x[4 * q + 1]), fmaxf(x[4 * q + 2], x[4 * q + 3]));
        b[q] = fmaxf(fmaxf(y[4 * q], y[4 * q + 1]), fmaxf(y[4 * q + 2], y[4 * q + 3]));
    }
    sort8_desc(a);
    sort8_desc(b);
    float t = INFINITY;
#pragma unroll
    for (int q = 0; q < 8; ++q) t = fminf(t, fmaxf(a[q], b[7 - q]));
    return t;
}
__device__ __forceinline__ int visible_in_block(int64_t nvis, int64_t c0) {
    const int64_t n = nvis - c0;
    return n <= 0 ? 0 : n >= 32 ? 32 : (int)n;
}
template <int KP>
__device__ __forceinline__ void topk_block(const float (&sc)[32], int64_t c0, int lim, float scale,
                                           TopList<KP> &v, float &tf, float *stage, int r,
                                           float floor) {
    // every bound is loosened by 1e-6 of its size: an unscaled score just
    // below a bound can round to the same scaled score as one at the bound
    // and then rank above it on its lower index, so it stays a candidate
    // (-inf stays -inf)
    const float tq = tf / scale;                                // scale > 0
    float tr = fmaxf(tq - fabsf(tq) * 1e-6f, floor - fabsf(floor) * 1e-6f);
    if (tr == -INFINITY && lim == 32 && KP < 32) {
        // empty list, full block: the smallest of the maxima of KP groups of
        // 32/KP columns is a lower bound on the KP-th largest of the 32 (each
        // group holds a score at or above it), so only scores at or above it
        // can enter; this keeps the first block from inserting every column
        constexpr int GS = 32 / (KP < 32 ? KP : 16);
        float bound = INFINITY;
#pragma unroll
        for (int g0 = 0; g0 < 32; g0 += GS) {
            float m = sc[g0];
#pragma unroll
            for (int c = 1; c < GS; ++c) m = fmaxf(m, sc[g0 + c]);
            bound = fminf(bound, m);
        }
        tr = bound - fabsf(bound) * 1e-6f;
    }
    uint32_t mask = 0;
#pragma unroll
    for (int c = 0; c < 32; ++c) mask |= (sc[c] >= tr ? 1u : 0u) << c;
    mask &= lim >= 32 ? 0xffffffffu : (1u << lim) - 1u;
    if (mask) {
#pragma unroll
        for (int c = 0; c < 32; ++c) stage[c * 128 + r] = sc[c];
    }
    // Branch-free trips: an entry below every held one leaves the list as it
    // is, so no score test is needed, and the threshold is refreshed once at
    // the end.
    while (mask) {
        const int c = __ffs(mask) - 1;
        mask &= mask - 1;
        v.insert_later(scale * stage[c * 128 + r], (int32_t)c0 + c);
    }
    tf = v.s[KP - 1];
}

// The top-K runs in two groups of four warps (thread = token = TMEM lane),
// each over alternate 32-column blocks of the scores into its own list;
// group 1 leaves its list in shared memory (`lists`: [KP][128] scores, then
// [KP][128] indices) and group 0 folds it into its own under the total order,
// so the result is the token's top K whatever the split.
template <int KP>
__device__ __forceinline__ void merge_lists(TopList<KP> &v, const float *lists, int r) {
    const int32_t *li = reinterpret_cast<const int32_t *>(lists + KP * 128);
#pragma unroll
    for (int j = 0; j < KP; ++j) {
        const int32_t xi = li[j * 128 + r];
        if (xi >= 0) v.insert_any(lists[j * 128 + r], xi);
    }
}

template <int D, bool LM32, int KP>
__global__ void __launch_bounds__(kSelTcThreads, 1)
select_tc_kernel(const __grid_constant__ CUtensorMap tmL0, const __grid_constant__ CUtensorMap tmL1,
                 const SelTcParams p) {
    using C = SelCfg<D, LM32>;
    grid_dep_wait();                      // landmarks may come from the previous kernels
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *sA = smem;                                        // [QP][KB][M x 128 B]
    auto sB = [&](int s) { return smem + C::QP * C::A_PART + s * C::B_STAGE; };   // [LP][KB][N x 128 B]
    uint64_t *bars = (uint64_t *)(smem + C::BAR_OFF);
    uint64_t *full = bars, *empty = bars + C::STAGES;                  // [STAGES]
    uint64_t *tfull = bars + 2 * C::STAGES, *tfree = tfull + 2;        // [2] TMEM slots
    uint32_t *s_tmem = (uint32_t *)(tfree + 2);
    static_assert((2 * C::STAGES + 4) * 8 + 8 <= 256, "barrier block overflows its reserve");
    volatile int *s_abort = (volatile int *)(s_tmem + 1);

    const int ntb = (int)((p.Lsel + C::M - 1) / C::M);
    const int tb = ntb - 1 - (int)blockIdx.x;                  // heavy blocks first
    const int64_t bg = blockIdx.y;
    const int64_t b = bg / p.Hkv;
    const int g = (int)(bg % p.Hkv);
    const int G = p.H / p.Hkv;
    const int64_t L = p.L, Lsel = p.Lsel;
    const int R = p.R;
    const int64_t t0 = (int64_t)tb * C::M;                     // first selection row
    const int64_t t_last = t0 + C::M - 1 < Lsel ? t0 + C::M - 1 : Lsel - 1;
    const int64_t nvis_max = chunk_of(p.ch, t_last * R);       // visible to the block's last row
    const int ntiles = (int)((nvis_max + C::N - 1) / C::N);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (warp == 1) {
        tc::tmem_alloc(s_tmem, C::TMEM_COLS);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            tc::mbar_init(&full[s], 1);
            tc::mbar_init(&empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            tc::mbar_init(&tfull[s], 1);
            tc::mbar_init(&tfree[s], 8);       // one arrive per top-K warp
        }
        *s_abort = 0;
        tc::fence_barrier_init();
    }
    // the first landmark tiles do not depend on qbar: start their loads now
    auto issue_tile = [&](int n) {
        const int s = n % C::STAGES;
        tc::mbar_expect_tx(&full[s], (uint32_t)C::B_STAGE);
        const int row0 = (int)(bg * p.Nc + (int64_t)n * C::N);
#pragma unroll
        for (int lp = 0; lp < C::LP; ++lp)
#pragma unroll
            for (int kb = 0; kb < C::KB; ++kb)
                tc::tma_load_2d(sB(s) + lp * C::B_PART + kb * (C::N * 128), lp ? &tmL1 : &tmL0,
                                &full[s], kb * 64, row0);
    };
    if (tid == 0)
        for (int n = 0; n < ntiles && n < C::STAGES; ++n) issue_tile(n);
    // qbar = (1/G) sum_h q_h, split into bf16 parts, 128-byte swizzled K-major.
    // A thread owns (token, 16-byte vector) pairs and keeps two pairs' loads of
    // eight heads in flight (G is a multiple of 8 on this path).
    {
        constexpr int VPR = D / 8;                            // 16-byte vectors per row
        constexpr int NPAIR = C::M * VPR;
        for (int e0 = tid; e0 < NPAIR; e0 += 2 * kSelTcThreads) {
            float acc[2][8], inv[2];
            const __nv_bfloat16 *qp[2];
            int npairs[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int e = e0 + u * kSelTcThreads;
                const int r = e / VPR, c = e % VPR;
                const int64_t t = t0 + r;
                const bool live = e < NPAIR && t < Lsel;
                npairs[u] = live ? qbar_pairs(p, G, t) : 0;
                inv[u] = live ? 1.f / (float)npairs[u] : 0.f;
                qp[u] = (const __nv_bfloat16 *)p.Q + ((b * L + (live ? t * R : 0)) * p.H + (int64_t)g * G) * D + c * 8;
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[u][i] = 0.f;
            }
            const int nmax = npairs[0] > npairs[1] ? npairs[0] : npairs[1];
            for (int h0 = 0; h0 < nmax; h0 += 8) {
                // pairs h0 .. h0+7: token h0 / G of the row, heads h0 % G ..
                const int64_t off = (int64_t)(h0 / G) * p.H * D + (int64_t)(h0 % G) * D;
                uint4 raw[2][8];
#pragma unroll
                for (int u = 0; u < 2; ++u)
#pragma unroll
                    for (int h = 0; h < 8; ++h)
                        raw[u][h] = h0 < npairs[u] ? ld_stream16(qp[u] + off + (int64_t)h * D) : make_uint4(0, 0, 0, 0);
#pragma unroll
                for (int u = 0; u < 2; ++u)
#pragma unroll
                    for (int h = 0; h < 8; ++h) {
                        float f[8];
                        Vec16<__nv_bfloat16>::unpack(raw[u][h], f);
#pragma unroll
                        for (int i = 0; i < 8; ++i) acc[u][i] += f[i];
                    }
            }
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int e = e0 + u * kSelTcThreads;
                if (e >= NPAIR) continue;
                const int r = e / VPR, c = e % VPR;
                const uint32_t off = (uint32_t)((c / 8) * (C::M * 128)) + tc::sw128_offset(r, c % 8);
                float x[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) x[i] = acc[u][i] * inv[u];
#pragma unroll
                for (int part = 0; part < C::QP; ++part) {
                    uint32_t w[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint32_t lo = bf16_bits_rn(x[2 * i]), hi = bf16_bits_rn(x[2 * i + 1]);
                        w[i] = lo | (hi << 16);
                        x[2 * i] -= __uint_as_float(lo << 16);
                        x[2 * i + 1] -= __uint_as_float(hi << 16);
                    }
                    *reinterpret_cast<uint4 *>(sA + part * C::A_PART + off) = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
        }
        tc::fence_proxy_async_smem();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *s_tmem;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            for (int n = C::STAGES; n < ntiles; ++n) {
                const int s = n % C::STAGES;
                if (!sel_wait(&empty[s], (uint32_t)(((n / C::STAGES) + 1) & 1), s_abort)) break;
                issue_tile(n);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC = tc::idesc_bf16_f32(128, C::N, false);
            // (qbar part, landmark part) of every product term
            constexpr int NPROD = 3;
            constexpr int pa[NPROD] = {0, 1, LM32 ? 0 : 2};
            constexpr int pl[NPROD] = {0, 0, LM32 ? 1 : 0};
            // descriptors built once; an operand offset moves only the start-
            // address field (bytes / 16, shared memory below 256 KB: no carry)
            const uint64_t ad0 = tc::sdesc_sw128(tc::smem_u32(sA), 16, 1024);
            const uint64_t bd0 = tc::sdesc_sw128(tc::smem_u32(sB(0)), 16, 1024);
            for (int n = 0; n < ntiles; ++n) {
                const int s = n % C::STAGES, ts = n & 1;          // landmark stage, TMEM slot
                if (!sel_wait(&full[s], (uint32_t)((n / C::STAGES) & 1), s_abort)) break;
                if (n >= 2 && !sel_wait(&tfree[ts], (uint32_t)(((n >> 1) + 1) & 1), s_abort)) break;
                tc::fence_after_sync();
                const uint64_t bds = bd0 + (uint64_t)(s * (C::B_STAGE / 16));
                const uint32_t dt = tmem + ts * C::N;
#pragma unroll
                for (int pr = 0; pr < NPROD; ++pr)
#pragma unroll
                    for (int kb = 0; kb < C::KB; ++kb)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            tc::mma_bf16(dt, ad0 + (uint64_t)((pa[pr] * C::A_PART + kb * (C::M * 128) + kk * 32) / 16),
                                         bds + (uint64_t)((pl[pr] * C::B_PART + kb * (C::N * 128) + kk * 32) / 16),
                                         IDESC, (pr | kb | kk) ? 1u : 0u);
                tc::mma_commit(&tfull[ts]);
                tc::mma_commit(&empty[s]);
            }
        }
    } else if (warp < 10) {
        // ------------------------------------------------------------ top-K
        // group 0 (warps 2-5) takes the 32-column blocks 0 and 2 of every
        // score tile, group 1 (warps 6-9) blocks 1 and 3 (see merge_lists)
        const int q4 = warp & 3;
        const int hg = (warp - 2) >> 2;
        const int r = q4 * 32 + lane;
        float *stage = (float *)(smem + C::STAGE_OFF) + hg * (32 * 128);
        const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
        const int64_t t = t0 + r;                              // selection row
        const int64_t nvis = t < Lsel ? chunk_of(p.ch, t * R) : 0;
        TopList<KP> v;
        v.clear();
        float tf = -INFINITY;                                  // score of v's K-th entry
        for (int n = 0; n < ntiles; ++n) {
            const int s = n & 1;
            // warp-uniform outcome: the TMEM loads below are .sync.aligned
            if (!__all_sync(0xffffffffu, sel_wait(&tfull[s], (uint32_t)((n >> 1) & 1), s_abort)))
                break;
            tc::fence_after_sync();
            // 32-column blocks past the block's last visible chunk hold nothing
            const int64_t vis = nvis_max - (int64_t)n * C::N;
            const int ncb = vis >= C::N ? C::N / 32 : (int)((vis + 31) / 32);
            // this group's two 32-column blocks (cb = hg, hg + 2): both loads
            // are issued before one wait
            if (hg < ncb) {
                float sc0[32], sc1[32];
                const bool two = hg + 2 < ncb;
                tc::tmem_ld32(tmem + s * C::N + hg * 32 + lane_off, sc0);
                if (two) tc::tmem_ld32(tmem + s * C::N + (hg + 2) * 32 + lane_off, sc1);
                tc::tmem_wait_ld();
                const int64_t c0 = (int64_t)n * C::N + hg * 32;
                const int lim0 = visible_in_block(nvis, c0);
                const int lim1 = two ? visible_in_block(nvis, c0 + 64) : 0;
                float floor = -INFINITY;
                if (KP == 8 && tf == -INFINITY && lim1 == 32) floor = eighth_bound64(sc0, sc1);
                topk_block<KP>(sc0, c0, lim0, p.scale, v, tf, stage, r, floor);
                if (two) topk_block<KP>(sc1, c0 + 64, lim1, p.scale, v, tf, stage, r, floor);
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&tfree[s]);
        }
        // the landmark stages are dead once the last tile's scores are in TMEM
        float *lists = reinterpret_cast<float *>(sB(0));
        if (hg == 1) {
#pragma unroll
            for (int k = 0; k < KP; ++k) {
                lists[k * 128 + r] = v.s[k];
                reinterpret_cast<int32_t *>(lists + KP * 128)[k * 128 + r] = v.i[k];
            }
        }
        asm volatile("bar.sync 1, 256;" ::: "memory");     // the two top-K groups
        if (hg == 0 && t < Lsel) {
            merge_lists<KP>(v, lists, r);
            // the row's selection serves its R tokens
            for (int j = 0; j < R && t * R + j < L; ++j) {
                int32_t *dst = p.idx + ((b * L + t * R + j) * p.Hkv + g) * p.topk;
#pragma unroll
                for (int k = 0; k < KP; ++k)
                    if (k < p.topk) dst[k] = v.i[k];
            }
        }
    } else if (R == 1) {
        // warps 10-11: warm L2 with the query rows of the block that will
        // most likely start on some SM a wave later (one block per SM, blocks
        // placed in launch order), so its qbar loads come from L2
        uint32_t nsm;
        asm("mov.u32 %0, %%nsmid;" : "=r"(nsm));
        const int64_t lin = (int64_t)blockIdx.y * gridDim.x + blockIdx.x + nsm;
        if (lin < (int64_t)gridDim.x * gridDim.y) {
            const int tbn = ntb - 1 - (int)(lin % gridDim.x);
            const int64_t bgn = lin / gridDim.x;
            const int64_t bn = bgn / p.Hkv;
            const int gn = (int)(bgn % p.Hkv);
            for (int rr = tid - 10 * 32; rr < C::M; rr += 64) {
                const int64_t t = (int64_t)tbn * C::M + rr;
                if (t < L) {
                    const __nv_bfloat16 *src = (const __nv_bfloat16 *)p.Q + ((bn * L + t) * p.H + (int64_t)gn * G) * D;
                    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"((uint32_t)(G * D * 2))
                                 : "memory");
                }
            }
        }
    }

    __syncthreads();
    if (*s_abort) {
        if (tid == 0) atomicOr(p.status, kFlagTimeout);
        const long long t1 = clock64();
        while (clock64() - t1 < 20000000) { }
    }
    tc::fence_after_sync();
    if (warp == 1) tc::tmem_dealloc(tmem, C::TMEM_COLS);
}

// ---------------------------------------------------------------- one score tile
// When every chunk fits one N-tile (Nc <= 128, i.e. L <= 8192 at S = 64), the
// block builds qbar one 64-column block of d at a time into the same buffer:
// the score MMAs of block kb run while nothing else waits on them, and the
// next block is written once they are done (`half` barrier).  With one
// landmark stage and one TMEM score slot the block needs about 80 KB (bf16
// landmarks) or 96 KB (fp32 landmarks) of shared memory and 256 threads of at
// most 128 registers, so two blocks share an SM: one block's loads of the
// query rows overlap the other's MMAs and top-K, and a 4 x 4096-token batch
// runs in a single wave.
template <int D, bool LM32>
struct SelHalfCfg {
    static constexpr int M = 128, N = 128, KB = D / 64;
    static constexpr int QP = LM32 ? 2 : 3;
    static constexpr int LP = LM32 ? 2 : 1;
    static constexpr int A_PART = M * 128;            // one 64-column block of qbar
    static constexpr int B_PART = N * D * 2;
    static constexpr int BAR_OFF = QP * A_PART + LP * B_PART;
    static constexpr int SMEM = 1024 + BAR_OFF + 256;
    static constexpr uint32_t TMEM_COLS = N;
    // the top-K score rows ([32][128] fp32) reuse the qbar buffer: the top-K
    // starts once the last score MMA, its last reader, has completed
    static_assert(QP * A_PART >= 32 * 128 * 4, "top-K rows must fit the qbar buffer");
};
constexpr int kSelHalfThreads = 256;                // 8 warps: all build qbar; 2-5 also top-K

template <int D, bool LM32, int KP>
__global__ void __launch_bounds__(kSelHalfThreads, 2)
select_tc_half_kernel(const __grid_constant__ CUtensorMap tmL0, const __grid_constant__ CUtensorMap tmL1,
                      const SelTcParams p) {
    using C = SelHalfCfg<D, LM32>;
    grid_dep_wait();                      // landmarks may come from the previous kernels
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *sA = smem;                                        // [QP][M x 128 B]
    uint8_t *sB = smem + C::QP * C::A_PART;                    // [LP][KB][N x 128 B]
    uint64_t *bars = (uint64_t *)(smem + C::BAR_OFF);
    uint64_t *full = bars, *half = bars + 1, *tfull = bars + 2;
    uint32_t *s_tmem = (uint32_t *)(bars + 3);
    volatile int *s_abort = (volatile int *)(s_tmem + 1);

    const int ntb = (int)((p.Lsel + C::M - 1) / C::M);
    const int tb = ntb - 1 - (int)blockIdx.x;                  // heavy blocks first
    const int64_t bg = blockIdx.y;
    const int64_t b = bg / p.Hkv;
    const int g = (int)(bg % p.Hkv);
    const int G = p.H / p.Hkv;
    const int64_t L = p.L, Lsel = p.Lsel;
    const int R = p.R;
    const int64_t t0 = (int64_t)tb * C::M;                     // first selection row
    const int64_t t_last = t0 + C::M - 1 < Lsel ? t0 + C::M - 1 : Lsel - 1;
    const int64_t nvis_max = chunk_of(p.ch, t_last * R);       // visible to the block's last row
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (warp == 1) {
        tc::tmem_alloc(s_tmem, C::TMEM_COLS);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        tc::mbar_init(full, 1);
        tc::mbar_init(half, 1);
        tc::mbar_init(tfull, 1);
        *s_abort = 0;
        tc::fence_barrier_init();
        // the landmark tile does not depend on qbar: start its loads now
        tc::mbar_expect_tx(full, (uint32_t)(C::LP * C::B_PART));
        const int row0 = (int)(bg * p.Nc);
#pragma unroll
        for (int lp = 0; lp < C::LP; ++lp)
#pragma unroll
            for (int kb = 0; kb < C::KB; ++kb)
                tc::tma_load_2d(sB + lp * C::B_PART + kb * (C::N * 128), lp ? &tmL1 : &tmL0, full,
                                kb * 64, row0);
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *s_tmem;
    bool ok = true;
    for (int kb = 0; kb < C::KB; ++kb) {
        if (kb > 0) {
            // the MMAs of block kb-1 are done reading the buffer
            ok = sel_wait(half, (uint32_t)((kb - 1) & 1), s_abort);
            if (!__syncthreads_and(ok)) break;
        }
        // qbar columns kb*64 .. +64: a thread owns (token, 16-byte vector)
        // pairs and keeps two pairs' loads of eight heads in flight
        constexpr int NPAIR = C::M * 8;
        for (int e0 = tid; e0 < NPAIR; e0 += 2 * kSelHalfThreads) {
            float acc[2][8], inv[2];
            const __nv_bfloat16 *qp[2];
            int npairs[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int e = e0 + u * kSelHalfThreads;
                const int r = e / 8, c = e % 8;
                const int64_t t = t0 + r;
                const bool live = e < NPAIR && t < Lsel;
                npairs[u] = live ? qbar_pairs(p, G, t) : 0;
                inv[u] = live ? 1.f / (float)npairs[u] : 0.f;
                qp[u] = (const __nv_bfloat16 *)p.Q + ((b * L + (live ? t * R : 0)) * p.H + (int64_t)g * G) * D +
                        kb * 64 + c * 8;
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[u][i] = 0.f;
            }
            const int nmax = npairs[0] > npairs[1] ? npairs[0] : npairs[1];
            for (int h0 = 0; h0 < nmax; h0 += 8) {
                const int64_t off = (int64_t)(h0 / G) * p.H * D + (int64_t)(h0 % G) * D;
                uint4 raw[2][8];
#pragma unroll
                for (int u = 0; u < 2; ++u)
#pragma unroll
                    for (int h = 0; h < 8; ++h)
                        raw[u][h] = h0 < npairs[u] ? ld_stream16(qp[u] + off + (int64_t)h * D) : make_uint4(0, 0, 0, 0);
#pragma unroll
                for (int u = 0; u < 2; ++u)
#pragma unroll
                    for (int h = 0; h < 8; ++h) {
                        float f[8];
                        Vec16<__nv_bfloat16>::unpack(raw[u][h], f);
#pragma unroll
                        for (int i = 0; i < 8; ++i) acc[u][i] += f[i];
                    }
            }
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int e = e0 + u * kSelHalfThreads;
                if (e >= NPAIR) continue;
                const int r = e / 8, c = e % 8;
                const uint32_t off = tc::sw128_offset(r, c);
                float x[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) x[i] = acc[u][i] * inv[u];
#pragma unroll
                for (int part = 0; part < C::QP; ++part) {
                    uint32_t w[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint32_t lo = bf16_bits_rn(x[2 * i]), hi = bf16_bits_rn(x[2 * i + 1]);
                        w[i] = lo | (hi << 16);
                        x[2 * i] -= __uint_as_float(lo << 16);
                        x[2 * i + 1] -= __uint_as_float(hi << 16);
                    }
                    *reinterpret_cast<uint4 *>(sA + part * C::A_PART + off) = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
        }
        tc::fence_proxy_async_smem();
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
        if (warp == 1 && lane == 0) {
            // the score products of this block of d (see SelCfg's split)
            constexpr uint32_t IDESC = tc::idesc_bf16_f32(128, C::N, false);
            constexpr int NPROD = 3;
            const int pa[NPROD] = {0, 1, LM32 ? 0 : 2};
            const int pl[NPROD] = {0, 0, LM32 ? 1 : 0};
            bool go = kb > 0 || sel_wait(full, 0u, s_abort);
            if (go) {
                tc::fence_after_sync();
#pragma unroll
                for (int pr = 0; pr < NPROD; ++pr)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t ad = tc::sdesc_sw128(tc::smem_u32(sA + pa[pr] * C::A_PART + kk * 32), 16, 1024);
                        const uint64_t bd = tc::sdesc_sw128(
                            tc::smem_u32(sB + pl[pr] * C::B_PART + kb * (C::N * 128) + kk * 32), 16, 1024);
                        tc::mma_bf16(tmem, ad, bd, IDESC, (kb | pr | kk) ? 1u : 0u);
                    }
                tc::mma_commit(kb + 1 < C::KB ? half : tfull);
            }
        }
    }
    if (warp >= 2 && warp < 6) {
        // ------------------------------------------------------------ top-K
        const int q4 = warp & 3;
        const int r = q4 * 32 + lane;
        const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
        const int64_t t = t0 + r;                              // selection row
        const int64_t nvis = t < Lsel ? chunk_of(p.ch, t * R) : 0;
        TopList<KP> v;
        v.clear();
        float tf = -INFINITY;                                  // score of v's K-th entry
        // warp-uniform outcome: the TMEM loads below are .sync.aligned
        if (__all_sync(0xffffffffu, ok && sel_wait(tfull, 0u, s_abort))) {
            tc::fence_after_sync();
            // 32-column blocks past the block's last visible chunk hold nothing
            const int ncb = nvis_max >= C::N ? C::N / 32 : (int)((nvis_max + 31) / 32);
            // two blocks' loads per wait where the registers allow (two blocks of
            // 32 scores next to a 16-key list stay within the 128 registers a
            // thread has at two blocks per SM)
            constexpr int STEP = KP <= 8 ? 2 : 1;
#pragma unroll 1
            for (int cb = 0; cb < ncb; cb += STEP) {
                float sc0[32], sc1[32];
                const bool two = STEP == 2 && cb + 1 < ncb;
                tc::tmem_ld32(tmem + cb * 32 + lane_off, sc0);
                if (two) tc::tmem_ld32(tmem + (cb + 1) * 32 + lane_off, sc1);
                tc::tmem_wait_ld();
                const int64_t c0 = (int64_t)cb * 32;
                const int lim0 = visible_in_block(nvis, c0);
                const int lim1 = two ? visible_in_block(nvis, c0 + 32) : 0;
                float floor = -INFINITY;
                if (KP == 8 && tf == -INFINITY && lim1 == 32) floor = eighth_bound64(sc0, sc1);
                topk_block<KP>(sc0, c0, lim0, p.scale, v, tf, (float *)sA, r, floor);
                if (two) topk_block<KP>(sc1, c0 + 32, lim1, p.scale, v, tf, (float *)sA, r, floor);
            }
            tc::fence_before_sync();
            for (int j = 0; j < R && t < Lsel && t * R + j < L; ++j) {
                int32_t *dst = p.idx + ((b * L + t * R + j) * p.Hkv + g) * p.topk;
#pragma unroll
                for (int k = 0; k < KP; ++k)
                    if (k < p.topk) dst[k] = v.i[k];
            }
        }
    }

    __syncthreads();
    if (*s_abort) {
        if (tid == 0) atomicOr(p.status, kFlagTimeout);
        const long long t1 = clock64();
        while (clock64() - t1 < 20000000) { }
    }
    tc::fence_after_sync();
    if (warp == 1) tc::tmem_dealloc(tmem, C::TMEM_COLS);
}

// fp32 landmarks -> two bf16 parts l0 = rn(x), l1 = rn(x - l0).
__global__ void __launch_bounds__(256)
split_landmarks_kernel(const float4 *__restrict__ lm, uint2 *__restrict__ l0, uint2 *__restrict__ l1,
                       int64_t n4) {
    grid_dep_wait();
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float4 x = lm[i];
        const float xs[4] = {x.x, x.y, x.z, x.w};
        uint32_t h[4], r[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            h[e] = bf16_bits_rn(xs[e]);
            r[e] = bf16_bits_rn(xs[e] - __uint_as_float(h[e] << 16));
        }
        l0[i] = make_uint2(h[0] | (h[1] << 16), h[2] | (h[3] << 16));
        l1[i] = make_uint2(r[0] | (r[1] << 16), r[2] | (r[3] << 16));
    }
}

// ---------------------------------------------------------------- host side
typedef CUresult (*SelEncodeFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static SelEncodeFn sel_encode_fn() {
    static SelEncodeFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            fn = (SelEncodeFn)ptr;
    }
    return fn;
}

// bf16 landmark rows [rows, D]: boxes of 64 columns x box_rows rows (one
// score tile's chunks), 128-byte swizzle; rows past the end read as zero.
static bool sel_make_map(CUtensorMap *m, const void *base, uint64_t rows, int D, int box_rows) {
    SelEncodeFn enc = sel_encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
    const cuuint32_t es[2] = {1u, 1u};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
               es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

template <int D, bool LM32, int KP>
static cudaError_t launch_select_tc_t(const SelTcParams &p, int B, const void *l0, const void *l1,
                                      bool force_multi_tile, bool *multi, cudaStream_t st) {
    using C = SelCfg<D, LM32>;
    const uint64_t rows = (uint64_t)B * p.Hkv * p.Nc;
    dim3 grid((unsigned)((p.Lsel + C::M - 1) / C::M), (unsigned)(B * p.Hkv));
    *multi = !(p.Nc <= SelHalfCfg<D, LM32>::N && !force_multi_tile);
    const int box_rows = *multi ? C::N : SelHalfCfg<D, LM32>::N;
    CUtensorMap m0, m1;
    if (!sel_make_map(&m0, l0, rows, D, box_rows)) return cudaErrorInvalidValue;
    if (LM32) {
        if (!sel_make_map(&m1, l1, rows, D, box_rows)) return cudaErrorInvalidValue;
    } else {
        m1 = m0;
    }
    if (!*multi) {
        // every chunk fits one score tile: qbar built per 64-column block, two blocks per SM
        using H = SelHalfCfg<D, LM32>;
        auto kern = select_tc_half_kernel<D, LM32, KP>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, H::SMEM);
        if (e != cudaSuccess) return e;
        return launch_pdl(kern, grid, dim3(kSelHalfThreads), (size_t)H::SMEM, st, m0, m1, p);
    }
    auto kern = select_tc_kernel<D, LM32, KP>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, grid, dim3(kSelTcThreads), (size_t)C::SMEM, st, m0, m1, p);
}

template <int D, bool LM32>
static cudaError_t launch_select_tc_k(const SelTcParams &p, int B, const void *l0, const void *l1,
                                      bool fm, bool *multi, cudaStream_t st) {
    if (p.topk <= 8) return launch_select_tc_t<D, LM32, 8>(p, B, l0, l1, fm, multi, st);
    if (p.topk <= 16) return launch_select_tc_t<D, LM32, 16>(p, B, l0, l1, fm, multi, st);
    return launch_select_tc_t<D, LM32, 32>(p, B, l0, l1, fm, multi, st);
}

bool select_tc_supported() { return sel_encode_fn() != nullptr; }

// fp32 landmarks [n] -> two bf16 planes: split = [hi (n) | lo (n)].
cudaError_t launch_split_landmarks(const void *lm, void *split, int64_t n, cudaStream_t st) {
    __nv_bfloat16 *l0 = (__nv_bfloat16 *)split, *l1 = l0 + n;
    const int64_t n4 = n / 4;
    const unsigned blocks = (unsigned)((n4 + 255) / 256 < 4096 ? (n4 + 255) / 256 : 4096);
    return launch_pdl(split_landmarks_kernel, dim3(blocks), dim3(256), 0, st,
                      (const float4 *)lm, (uint2 *)l0, (uint2 *)l1, n4);
}

// Q bf16; landmarks bf16 (lm_bf16), else the two bf16 planes `split` of fp32
// landmarks (launch_split_landmarks, B*Hkv*Nc*d elements each).  Nc = L / S
// >= 1; G = H / Hkv a multiple of 8.  Up to 128 chunks the one-tile kernel
// runs unless `force_multi_tile`; `*multi` tells which kernel was launched.
cudaError_t launch_select_tc(const void *Q, const void *lm, bool lm_bf16, const void *split, int B,
                             int H, int Hkv, int64_t L, int d, int S, int64_t Nc, int topk,
                             float scale, int R, int pool_mean, const int32_t *bounds,
                             const int32_t *tok_chunk, int32_t *idx, unsigned *status,
                             bool force_multi_tile, bool *multi, cudaStream_t st) {
    SelTcParams p;
    p.Q = Q; p.idx = idx; p.status = status;
    p.L = L; p.Nc = Nc; p.H = H; p.Hkv = Hkv; p.S = S; p.topk = topk; p.scale = scale;
    p.R = R; p.pool_mean = pool_mean; p.Lsel = (L + R - 1) / R;
    p.ch.bounds = bounds; p.ch.tok_chunk = tok_chunk; p.ch.L = L; p.ch.S = S;
    const bool fm = force_multi_tile;
    if (lm_bf16) {
        return d == 128 ? launch_select_tc_k<128, false>(p, B, lm, nullptr, fm, multi, st)
                        : launch_select_tc_k<64, false>(p, B, lm, nullptr, fm, multi, st);
    }
    const int64_t n = (int64_t)B * Hkv * p.Nc * d;
    const __nv_bfloat16 *l0 = (const __nv_bfloat16 *)split, *l1 = l0 + n;
    return d == 128 ? launch_select_tc_k<128, true>(p, B, l0, l1, fm, multi, st)
                    : launch_select_tc_k<64, true>(p, B, l0, l1, fm, multi, st);
}

}  // namespace hsa
