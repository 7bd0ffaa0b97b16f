// attend_tc.cu -- in-chunk attention on the 5th-generation tensor cores
// (tcgen05 MMA, TMEM accumulators, TMA tile loads), bf16 in, fp32 accumulate,
// and the score-weighted fusion of the chunk outputs.
//
// HiLS Attention abstract: every query attends independently inside each
// retrieved chunk; the chunk outputs are fused with weights from the retrieval
// scores.  The work is chunk-bucketed (bucket.cu): a tile is one chunk's 64
// keys/values plus up to 128/G selected entries, each entry contributing its G
// query-head rows (the heads of a KV group share the selection), so a tile is a
// dense 128-row problem.  The chunk's landmark rides along as two extra "key"
// rows (its bf16 high and low parts), so the same MMA also yields every row's
// fusion logit scale * q_h . l_chunk:
//
//   S = Q_rows . [K_chunk ; l_hi ; l_lo]^T  M=128, N=80, K=d  (tcgen05 -> TMEM)
//   P = exp(S*scale - rowmax) / rowsum      per row in registers, bf16 -> smem
//   O = P . V_chunk                         M=128, N=d, K=64  (tcgen05 -> TMEM)
//   partial[t, g, k] = O (fp16), logit[t, h, k] = scale * (S[:,64] + S[:,65])
//
// Own tiles: 128/G consecutive tokens of a chunk against that chunk with the
// causal mask (keys c*S .. t); their output (the own-chunk term) goes to an
// fp16 array.  fuse_kernel then completes the method, one warp per (t, h):
//   w = softmax over the token's selected chunks of the logits,
//   O = own_term + sum_k w_k * partial_k  (bf16 out).
//
// attend_tc_kernel: one persistent block per SM walks the tile queue with
// four roles linked by mbarriers and double-buffered shared memory / TMEM:
//   warp 0      producer  (tile metadata into a shared ring, landmark rows
//                          into smem, TMA of the chunk's K and V)
//   warp 10     Q gather  (one TMA box per entry: its G query-head rows)
//   warp 1      MMA issuer (S of the next tile or P.V of the oldest pending
//                          one, whichever is ready)
//   warps 2-5   softmax   (thread = tile row = TMEM lane)
//   warps 6-9   epilogue  (TMEM -> fp16 partial slots / own-chunk term)
// Tiles are independent, so no block waits on another.  Every wait is
// bounded; on expiry the block sets the status flag in the workspace, lets
// in-flight copies land, frees its TMEM and exits.
#include <cuda.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "tc.cuh"

namespace hsa {

template <int D, int G>
struct TcCfg {
    static constexpr int M = 128;
    static constexpr int EPT = M / G;            // entries (or tokens) per tile
    static constexpr int KB = D / 64;            // 64-element blocks of d
    static constexpr int NS = 80;                // S columns: 64 keys, l_hi, l_lo, pad
    static constexpr int Q_BYTES = M * D * 2;    // gathered query rows
    static constexpr int KBLK = NS * 128;        // one 64-wide d block of [K; l]
    static constexpr int K_BYTES = KB * KBLK;
    static constexpr int V_BYTES = 64 * D * 2;
    static constexpr int P_BYTES = M * 64 * 2;   // probabilities, bf16
    static constexpr int STAGE = Q_BYTES + K_BYTES + V_BYTES + P_BYTES;
    static constexpr int SMEM = 1024 + 2 * STAGE + 256;
    // TMEM: S[2] at columns 0 / 128 (80 used), O[2] at 256 / 256 + D
    static constexpr uint32_t S_COL = 128;
    static constexpr uint32_t O_COL = 256;
    static constexpr uint32_t TMEM_COLS = 512;
};

struct TcParams {
    const int64_t *seg_start;     // [2 * NW + 1]
    const int4 *wtiles;           // [NW * cap] retrieved-chunk tiles per window
    const int32_t *entries;
    const void *lm;               // [B, Hkv, Nc, D] bf16 or fp32
    float *logits;                // [B, L, H, topk] fusion logits
    __half *part;                 // [B*L*Hkv*topk entries][D/32][G][32] chunk outputs
    __half *own;                  // [B, L, H, D] own-chunk term
    unsigned *status;
    int64_t L, W, nwb, NW, cap, Nc;
    int H, Hkv, topk, S, add_own, lm_bf16;
    int q3d;                      // Q map is the 3-D (cols, rows, d-half) view
    float scale, scale_log2e;
};

constexpr long long kWaitBudget = 4000000000LL;    // SM cycles (about 2 s)
constexpr int kThreads = 352;                       // 11 warps
constexpr int kGatherWarp = 10;
constexpr int kMaxWindows = 2048;                  // shared segment table size / 2

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}
__device__ __forceinline__ uint32_t pack_f16x2(float a, float b) {
    __half2 v = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Bounded mbarrier wait that also gives up when another role aborted.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort) {
    if (tc::mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!tc::mbar_try_wait(bar, parity)) {
        if (*abort || clock64() - t0 > kWaitBudget) {
            *abort = 1;
            return false;
        }
    }
    return true;
}

// A queue position decoded into one tile.
struct Tile {
    int64_t bg, first, t0;   // first entry (retrieved) or first token (own)
    int chunk, n, own;
    int64_t win;
};

__device__ __forceinline__ void decode_tile(const TcParams &p, const int64_t *seg, int nseg,
                                            int64_t pos, int ept, Tile &tl) {
    int lo = 0, hi = nseg;                  // seg[lo] <= pos < seg[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (seg[mid] <= pos) lo = mid; else hi = mid;
    }
    const int64_t j = pos - seg[lo];
    if (lo == 0) { tl.own = 0; tl.win = 0; }
    else if (lo == nseg - 1) { tl.own = 1; tl.win = p.NW - 1; }
    else if (lo & 1) { tl.own = 0; tl.win = (lo + 1) / 2; }
    else { tl.own = 1; tl.win = lo / 2 - 1; }
    if (!tl.own) {
        const int4 d = p.wtiles[tl.win * p.cap + j];
        tl.bg = d.x; tl.chunk = d.y; tl.first = d.z; tl.n = d.w; tl.t0 = 0;
    } else {
        tl.bg = tl.win / p.nwb;
        const int64_t ts = (tl.win % p.nwb) * p.W;
        const int64_t te = ts + p.W < p.L ? ts + p.W : p.L;
        tl.t0 = ts + j * ept;
        tl.n = (int)(te - tl.t0 < ept ? te - tl.t0 : ept);
        tl.chunk = (int)(tl.t0 / p.S);
        tl.first = 0;
    }
}

// Tile metadata the producer publishes to the softmax and epilogue roles
// through a small shared-memory ring (so only the producer walks the global
// work lists).  code[e] = t * 32 + k of entry e (own tiles: t * 32).
constexpr int kRing = 4;
struct TileInfo {
    int64_t bg, win;
    int chunk, n, own, pad;
    int32_t code[16];
};

// Per-row view of a tile for the softmax and epilogue threads.
struct RowJob {
    Tile tl;
    int64_t t;
    int k;
    bool valid;
};

__device__ __forceinline__ RowJob read_row(const TileInfo &ti, int e) {
    RowJob rj;
    rj.tl.bg = ti.bg; rj.tl.win = ti.win; rj.tl.chunk = ti.chunk; rj.tl.n = ti.n;
    rj.tl.own = ti.own; rj.tl.first = 0; rj.tl.t0 = 0;
    rj.valid = e < ti.n;
    const int32_t code = rj.valid ? ti.code[e] : 0;
    rj.t = code >> 5;
    rj.k = code & 31;
    return rj;
}

template <int D, int G>
__global__ void __launch_bounds__(kThreads, 1)
attend_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const TcParams p) {
    using C = TcCfg<D, G>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    // stage s: [Q | K;l | V | P]
    auto sQ = [&](int s) { return smem + s * C::STAGE; };
    auto sK = [&](int s) { return smem + s * C::STAGE + C::Q_BYTES; };
    auto sV = [&](int s) { return smem + s * C::STAGE + C::Q_BYTES + C::K_BYTES; };
    auto sP = [&](int s) { return smem + s * C::STAGE + C::Q_BYTES + C::K_BYTES + C::V_BYTES; };
    uint64_t *bars = (uint64_t *)(smem + 2 * C::STAGE);
    uint64_t *full = bars, *empty = bars + 2, *sfull = bars + 4, *sfree = bars + 6;
    uint64_t *pfull = bars + 8, *ofull = bars + 10, *ofree = bars + 12;
    uint64_t *ifull = bars + 14, *ifree = bars + 14 + kRing;
    uint32_t *s_tmem = (uint32_t *)(bars + 14 + 2 * kRing);
    volatile int *s_abort = (volatile int *)(s_tmem + 1);
    __shared__ int64_t seg[2 * kMaxWindows + 1];
    __shared__ TileInfo ring[kRing];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nseg = (int)(2 * p.NW);
    for (int i = tid; i <= nseg; i += kThreads) seg[i] = p.seg_start[i];
    if (warp == 1) {
        tc::tmem_alloc(s_tmem, C::TMEM_COLS);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            tc::mbar_init(&full[s], 2);        // K/V producer + Q gather warp
            tc::mbar_init(&empty[s], 1);
            tc::mbar_init(&sfull[s], 1);
            tc::mbar_init(&sfree[s], 128);
            tc::mbar_init(&pfull[s], 128);
            tc::mbar_init(&ofull[s], 1);
            tc::mbar_init(&ofree[s], 128);
        }
        for (int i = 0; i < kRing; ++i) {
            tc::mbar_init(&ifull[i], 1);
            tc::mbar_init(&ifree[i], 257);     // softmax + epilogue threads + gather warp
        }
        *s_abort = 0;
        tc::fence_barrier_init();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *s_tmem;
    const int64_t qlen = seg[nseg];
    const int64_t L = p.L;
    const int H = p.H, Hkv = p.Hkv, topk = p.topk, S = p.S;
    constexpr int EPT = C::EPT;
    const int64_t my_tiles = qlen > blockIdx.x ? (qlen - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        // Software-pipelined two tiles deep: in iteration j the descriptor of
        // tile j+2 and the entry codes / landmark row of tile j+1 are loaded
        // while tile j is published and its copies are issued.
        auto load_rows = [&](const Tile &tl, int32_t &code, float (&x)[8]) {
            code = 0;
            if (lane < tl.n)
                code = tl.own ? (int32_t)((tl.t0 + lane) * 32) : p.entries[tl.first + lane];
            if (!tl.own && lane < D / 8) {
                const int64_t li = (tl.bg * p.Nc + tl.chunk) * D + lane * 8;
                if (p.lm_bf16) {
                    Vec16<__nv_bfloat16>::unpack(
                        *reinterpret_cast<const uint4 *>((const __nv_bfloat16 *)p.lm + li), x);
                } else {
                    const uint4 *src = reinterpret_cast<const uint4 *>((const float *)p.lm + li);
                    Vec16<float>::unpack(src[0], x);
                    Vec16<float>::unpack(src[1], x + 4);
                }
            }
        };
        Tile d0, d1;
        int32_t c0 = 0;
        float x0[8];
        if (my_tiles > 0) decode_tile(p, seg, nseg, blockIdx.x, EPT, d0);
        if (my_tiles > 1) decode_tile(p, seg, nseg, blockIdx.x + gridDim.x, EPT, d1);
        if (my_tiles > 0) load_rows(d0, c0, x0);
        for (int64_t j = 0; j < my_tiles; ++j) {
            Tile d2;
            if (j + 2 < my_tiles) decode_tile(p, seg, nseg, blockIdx.x + (j + 2) * gridDim.x, EPT, d2);
            int32_t c1 = 0;
            float x1[8];
            if (j + 1 < my_tiles) load_rows(d1, c1, x1);

            // publish the tile's metadata
            const int ri = (int)(j & (kRing - 1));
            int ok = 1;
            if (lane == 0 && j >= kRing)
                ok = wait_bar(&ifree[ri], (uint32_t)(((j / kRing) + 1) & 1), s_abort);
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            if (lane < 16) ring[ri].code[lane] = c0;
            if (lane == 0) {
                ring[ri].bg = d0.bg; ring[ri].win = d0.win; ring[ri].chunk = d0.chunk;
                ring[ri].n = d0.n; ring[ri].own = d0.own;
            }
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&ifull[ri]);

            // stage the tile's operands
            const int s = (int)(j & 1);
            if (lane == 0 && j >= 2) ok = wait_bar(&empty[s], (uint32_t)(((j >> 1) + 1) & 1), s_abort);
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            if (!d0.own && lane < D / 8) {
                // landmark row of the chunk -> key rows 64 (bf16 high part), 65 (low part)
                float hi[8], lo[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    hi[q] = __bfloat162float(__float2bfloat16_rn(x0[q]));
                    lo[q] = x0[q] - hi[q];
                }
                const int kb = (lane * 8) / 64, c = ((lane * 8) % 64) / 8;
                uint8_t *blk = sK(s) + kb * C::KBLK;
                *reinterpret_cast<uint4 *>(blk + tc::sw128_offset(64, c)) =
                    make_uint4(pack_bf16x2(hi[0], hi[1]), pack_bf16x2(hi[2], hi[3]),
                               pack_bf16x2(hi[4], hi[5]), pack_bf16x2(hi[6], hi[7]));
                *reinterpret_cast<uint4 *>(blk + tc::sw128_offset(65, c)) =
                    make_uint4(pack_bf16x2(lo[0], lo[1]), pack_bf16x2(lo[2], lo[3]),
                               pack_bf16x2(lo[4], lo[5]), pack_bf16x2(lo[6], lo[7]));
                tc::fence_proxy_async_smem();
            }
            __syncwarp();
            if (lane == 0) {
                // K and V of the chunk by TMA (the Q rows come from the gather warp)
                tc::mbar_expect_tx(&full[s], (uint32_t)(2 * C::V_BYTES));
                const int krow = (int)(d0.bg * L + (int64_t)d0.chunk * S);
#pragma unroll
                for (int kb = 0; kb < C::KB; ++kb) {
                    tc::tma_load_2d(sK(s) + kb * C::KBLK, &tmK, &full[s], kb * 64, krow);
                    tc::tma_load_2d(sV(s) + kb * 8192, &tmV, &full[s], kb * 64, krow);
                }
            }
            d0 = d1;
            d1 = d2;
            c0 = c1;
#pragma unroll
            for (int q = 0; q < 8; ++q) x0[q] = x1[q];
        }
    } else if (warp == kGatherWarp) {
        // ------------------------------------------------------------ Q gather
        // One TMA box per entry: all G query-head rows of the entry (both
        // 64-wide halves of d in one box when the 3-D view is available).
        for (int64_t j = 0; j < my_tiles; ++j) {
            const int ri = (int)(j & (kRing - 1));
            const int s = (int)(j & 1);
            int ok = 1;
            if (lane == 0) {
                ok = wait_bar(&ifull[ri], (uint32_t)((j / kRing) & 1), s_abort);
                if (ok && j >= 2) ok = wait_bar(&empty[s], (uint32_t)(((j >> 1) + 1) & 1), s_abort);
            }
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            const TileInfo &ti = ring[ri];
            const int n = ti.n;
            const int64_t b = ti.bg / Hkv;
            const int g = (int)(ti.bg % Hkv);
            const int32_t code = lane < n ? ti.code[lane] : 0;
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&ifree[ri]);
            if (lane == 0) tc::mbar_expect_tx(&full[s], (uint32_t)(n * G * D * 2));
            __syncwarp();
            if (lane < n) {
                const int qrow = (int)((b * L + (int64_t)(code >> 5)) * H + (int64_t)g * G);
                if (p.q3d) {
                    tc::tma_load_3d(sQ(s) + lane * (C::KB * G * 128), &tmQ, &full[s], 0, qrow, 0);
                } else {
#pragma unroll
                    for (int kb = 0; kb < C::KB; ++kb)
                        tc::tma_load_2d(sQ(s) + kb * (128 * 128) + lane * G * 128, &tmQ, &full[s],
                                        kb * 64, qrow);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC_S = tc::idesc_bf16_f32(128, C::NS, false);
            constexpr uint32_t IDESC_O = tc::idesc_bf16_f32(128, D, true);
            auto issue_pv = [&](int64_t i) {
                const int s = (int)(i & 1);
                tc::fence_after_sync();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t ad = tc::sdesc_sw128(tc::smem_u32(sP(s) + kk * 32), 16, 1024);
                    const uint64_t bd = tc::sdesc_sw128(tc::smem_u32(sV(s) + kk * 2048), 8192, 1024);
                    tc::mma_bf16(tmem + C::O_COL + s * D, ad, bd, IDESC_O, kk ? 1u : 0u);
                }
                tc::mma_commit(&ofull[s]);
                tc::mma_commit(&empty[s]);
            };
            // Issue S of the next tile or P.V of the oldest pending one, whichever
            // is ready first (at most two tiles in flight, one per stage).
            auto issue_s = [&](int64_t j) {
                const int s = (int)(j & 1);
                tc::fence_after_sync();
#pragma unroll
                for (int kb = 0; kb < C::KB; ++kb)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t ad = p.q3d
                            ? tc::sdesc_sw128(tc::smem_u32(sQ(s) + kb * (G * 128) + kk * 32), 16, C::KB * G * 128)
                            : tc::sdesc_sw128(tc::smem_u32(sQ(s) + kb * 16384 + kk * 32), 16, 1024);
                        const uint64_t bd = tc::sdesc_sw128(tc::smem_u32(sK(s) + kb * C::KBLK + kk * 32), 16, 1024);
                        tc::mma_bf16(tmem + s * C::S_COL, ad, bd, IDESC_S, (kb | kk) ? 1u : 0u);
                    }
                tc::mma_commit(&sfull[s]);
            };
            auto ready_s = [&](int64_t j) -> bool {
                const int s = (int)(j & 1);
                return tc::mbar_try_wait(&full[s], (uint32_t)((j >> 1) & 1)) &&
                       (j < 2 || tc::mbar_try_wait(&sfree[s], (uint32_t)(((j >> 1) + 1) & 1)));
            };
            auto ready_pv = [&](int64_t i) -> bool {
                const int s = (int)(i & 1);
                return tc::mbar_try_wait(&pfull[s], (uint32_t)((i >> 1) & 1)) &&
                       (i < 2 || tc::mbar_try_wait(&ofree[s], (uint32_t)(((i >> 1) + 1) & 1)));
            };
            int64_t ns = 0, npv = 0;
            long long t0 = clock64();
            while (npv < my_tiles) {
                if (ns < my_tiles && ns - npv < 2 && ready_s(ns)) {
                    issue_s(ns++);
                    t0 = clock64();
                } else if (npv < ns && ready_pv(npv)) {
                    issue_pv(npv++);
                    t0 = clock64();
                } else if (*s_abort || clock64() - t0 > kWaitBudget) {
                    *s_abort = 1;
                    break;
                }
            }
        }
    } else if (warp < 6) {
        // ------------------------------------------------------------ softmax
        const int q4 = warp & 3;                  // TMEM lane quarter
        const int r = q4 * 32 + lane;             // tile row
        const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
        const int e = r / G, h = r % G;
        for (int64_t j = 0; j < my_tiles; ++j) {
            const int ri = (int)(j & (kRing - 1));
            if (!wait_bar(&ifull[ri], (uint32_t)((j / kRing) & 1), s_abort)) break;
            const RowJob cur = read_row(ring[ri], e);
            tc::mbar_arrive(&ifree[ri]);
            const int s = (int)(j & 1);
            const int64_t b = cur.tl.bg / Hkv;
            const int g = (int)(cur.tl.bg % Hkv);
            if (!wait_bar(&sfull[s], (uint32_t)((j >> 1) & 1), s_abort)) break;
            tc::fence_after_sync();
            float s0[32], s1[32], l_hi, l_lo;
            const uint32_t ta = tmem + s * C::S_COL + lane_off;
            tc::tmem_ld32(ta, s0);
            tc::tmem_ld32(ta + 32, s1);
            tc::tmem_ld2(ta + 64, l_hi, l_lo);
            tc::tmem_wait_ld();
            tc::fence_before_sync();
            tc::mbar_arrive(&sfree[s]);
            if (cur.valid && !cur.tl.own)
                p.logits[((b * L + cur.t) * H + (int64_t)g * G + h) * topk + cur.k] =
                    p.scale * (l_hi + l_lo);
            const int nk = (cur.tl.own && cur.valid) ? (int)(cur.t - (int64_t)cur.tl.chunk * S) + 1 : 64;
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                if (c < nk) mx = fmaxf(mx, s0[c]);
                if (c + 32 < nk) mx = fmaxf(mx, s1[c]);
            }
            const float ms = mx * p.scale_log2e;
            float l = 0.f;
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                s0[c] = c < nk ? tc::ex2_approx(fmaf(s0[c], p.scale_log2e, -ms)) : 0.f;
                s1[c] = c + 32 < nk ? tc::ex2_approx(fmaf(s1[c], p.scale_log2e, -ms)) : 0.f;
                l += s0[c] + s1[c];
            }
            const float f = cur.valid ? (cur.tl.own ? (float)p.add_own : 1.f) / l : 0.f;
            if (j >= 2 && !wait_bar(&empty[s], (uint32_t)(((j >> 1) + 1) & 1), s_abort)) break;
            uint8_t *prow = sP(s);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const float *src = c < 4 ? s0 + 8 * c : s1 + 8 * (c - 4);
                const uint4 u = make_uint4(pack_bf16x2(src[0] * f, src[1] * f),
                                           pack_bf16x2(src[2] * f, src[3] * f),
                                           pack_bf16x2(src[4] * f, src[5] * f),
                                           pack_bf16x2(src[6] * f, src[7] * f));
                *reinterpret_cast<uint4 *>(prow + tc::sw128_offset(r, c)) = u;
            }
            tc::fence_proxy_async_smem();
            tc::mbar_arrive(&pfull[s]);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q4 = warp & 3;
        const int r = q4 * 32 + lane;
        const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
        const int e = r / G, h = r % G;
        constexpr int NCH = D / 32;               // 32-column chunks of a row
        for (int64_t j = 0; j < my_tiles; ++j) {
            const int ri = (int)(j & (kRing - 1));
            if (!wait_bar(&ifull[ri], (uint32_t)((j / kRing) & 1), s_abort)) break;
            const RowJob cur = read_row(ring[ri], e);
            tc::mbar_arrive(&ifree[ri]);
            const int s = (int)(j & 1);
            const int64_t b = cur.tl.bg / Hkv;
            const int g = (int)(cur.tl.bg % Hkv);
            const int64_t row = (b * L + cur.t) * Hkv + g;       // (t, g) selection row
            const int64_t hrow = (b * L + cur.t) * H + (int64_t)g * G + h;
            if (!wait_bar(&ofull[s], (uint32_t)((j >> 1) & 1), s_abort)) break;
            tc::fence_after_sync();
#pragma unroll 1
            for (int ch = 0; ch < NCH; ch += 2) {
                float o[2][32];
                // two 32-column TMEM loads per wait
                tc::tmem_ld32(tmem + C::O_COL + s * D + ch * 32 + lane_off, o[0]);
                tc::tmem_ld32(tmem + C::O_COL + s * D + (ch + 1) * 32 + lane_off, o[1]);
                tc::tmem_wait_ld();
                if (!cur.valid) continue;
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    // retrieved chunk: slot [entry][d/32][head][32]; own chunk: [t, h, d]
                    __half *dst = cur.tl.own
                        ? p.own + hrow * D + (ch + u) * 32
                        : p.part + (((row * topk + cur.k) * NCH + ch + u) * G + h) * 32;
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        reinterpret_cast<uint4 *>(dst)[q] = make_uint4(
                            pack_f16x2(o[u][8 * q + 0], o[u][8 * q + 1]), pack_f16x2(o[u][8 * q + 2], o[u][8 * q + 3]),
                            pack_f16x2(o[u][8 * q + 4], o[u][8 * q + 5]), pack_f16x2(o[u][8 * q + 6], o[u][8 * q + 7]));
                }
            }
            tc::fence_before_sync();
            tc::mbar_arrive(&ofree[s]);
        }
    }

    __syncthreads();
    if (*s_abort) {
        if (tid == 0) atomicOr(p.status, kFlagTimeout);
        // let copies and MMAs that may still be in flight land before exiting
        const long long t0 = clock64();
        while (clock64() - t0 < 20000000) { }
    }
    tc::fence_after_sync();
    if (warp == 1) tc::tmem_dealloc(tmem, C::TMEM_COLS);
}

// ---------------------------------------------------------------- fusion
// One warp per (t, h) row: w = softmax over the selected chunks of the
// logits, O = own + sum_k w_k * partial_k.  Lane l holds the D/32 consecutive
// elements d = l*D/32 ..; in the partial layout these are chunk l/(32/NCH),
// offset (l % (32/NCH)) * D/32 -- the same d.  Slot loads are unrolled so
// several are in flight.
template <int D, int G>
__global__ void __launch_bounds__(256)
fuse_kernel(const __half *__restrict__ part, const __half *__restrict__ own,
            const float *__restrict__ logits, const int32_t *__restrict__ idx, int64_t rows, int H,
            int Hkv, int topk, float *__restrict__ w_out, __nv_bfloat16 *__restrict__ O) {
    constexpr int EPL = D / 32;                      // elements per lane (4 or 2)
    constexpr int NCH = D / 32;                      // 32-wide chunks of d
    constexpr int LPC = 32 / NCH;                    // lanes per chunk
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    if (row >= rows) return;
    const int64_t bt = row / H;
    const int hh = (int)(row % H);
    const int g = hh / G, h = hh % G;
    const int64_t srow = bt * Hkv + g;               // selection row (t, g)
    const int32_t ik = lane < topk ? idx[srow * topk + lane] : -1;
    const int nsel = __popc(__ballot_sync(0xffffffffu, ik >= 0));   // valid slots come first
    const float lg = lane < nsel ? logits[row * topk + lane] : -INFINITY;
    float m = lg;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float ex = lane < nsel ? __expf(lg - m) : 0.f;
    float den = ex;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    const float w = nsel ? ex / den : 0.f;
    if (w_out && lane < topk) w_out[row * topk + lane] = w;

    const int ch = lane / LPC, off = (lane % LPC) * EPL;
    float acc[EPL];
    {
        const __half2 *s2 = reinterpret_cast<const __half2 *>(own + row * D + lane * EPL);
#pragma unroll
        for (int q = 0; q < EPL / 2; ++q) {
            const float2 v = __half22float2(s2[q]);
            acc[2 * q] = v.x;
            acc[2 * q + 1] = v.y;
        }
    }
    const __half *pbase = part + (((srow * topk) * NCH + ch) * G + h) * 32 + off;
    const int64_t kstride = (int64_t)NCH * G * 32;   // halves between slots k and k+1
#pragma unroll 8
    for (int k = 0; k < nsel; ++k) {
        const float wk = __shfl_sync(0xffffffffu, w, k);
        const __half2 *s2 = reinterpret_cast<const __half2 *>(pbase + k * kstride);
#pragma unroll
        for (int q = 0; q < EPL / 2; ++q) {
            const float2 v = __half22float2(s2[q]);
            acc[2 * q] = fmaf(wk, v.x, acc[2 * q]);
            acc[2 * q + 1] = fmaf(wk, v.y, acc[2 * q + 1]);
        }
    }
    __nv_bfloat162 *dst = reinterpret_cast<__nv_bfloat162 *>(O + row * D + lane * EPL);
#pragma unroll
    for (int q = 0; q < EPL / 2; ++q) dst[q] = __floats2bfloat162_rn(acc[2 * q], acc[2 * q + 1]);
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)ptr;
    }
    return fn;
}

// 2D bf16 view [rows, D] with 128-byte swizzled boxes of 64 columns x box_rows.
static bool make_map(CUtensorMap *m, const void *base, uint64_t rows, int D, int box_rows) {
    EncodeTiledFn enc = encode_fn();
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

// 3-D bf16 view of [rows, D] (D = 128) as (64 columns, rows, 2 halves of d),
// strides 2*D and 128 bytes: one box (64, G, 2) brings all of an entry's G
// rows, both halves, as two 128B-swizzled [G x 128 B] blocks.
static bool make_map_q3d(CUtensorMap *m, const void *base, uint64_t rows, int D, int G) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {64u, (cuuint64_t)rows, (cuuint64_t)(D / 64)};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 2, 128u};
    const cuuint32_t box[3] = {64u, (cuuint32_t)G, (cuuint32_t)(D / 64)};
    const cuuint32_t es[3] = {1u, 1u, 1u};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
               es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

struct TcLaunch {
    const void *Q, *K, *V, *lm;
    int B, H, Hkv, S, topk, own_chunk, lm_bf16;
    int64_t L, W, cap;
    float scale;
    const int32_t *idx, *entries;
    const int4 *wtiles;
    const int64_t *seg_start;
    float *logits, *w_out;
    __half *part, *own;
    void *O;
    unsigned *status;
    int num_sms;
};

template <int D, int G>
static cudaError_t launch_attend_tc_t(const TcLaunch &a, cudaStream_t st) {
    using C = TcCfg<D, G>;
    CUtensorMap mq, mk, mv;
    // the single-box entry layout has a uniform 8-row atom stride only when an
    // entry is exactly one atom (G = 8) and d has two halves
    bool q3d = (G == 8 && D == 128) &&
               make_map_q3d(&mq, a.Q, (uint64_t)a.B * a.L * a.H, D, G);
    if (!q3d && !make_map(&mq, a.Q, (uint64_t)a.B * a.L * a.H, D, G)) return cudaErrorInvalidValue;
    if (!make_map(&mk, a.K, (uint64_t)a.B * a.Hkv * a.L, D, 64) ||
        !make_map(&mv, a.V, (uint64_t)a.B * a.Hkv * a.L, D, 64))
        return cudaErrorInvalidValue;
    auto kern = attend_tc_kernel<D, G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    TcParams p;
    p.seg_start = a.seg_start; p.wtiles = a.wtiles;
    p.entries = a.entries; p.lm = a.lm; p.logits = a.logits;
    p.part = a.part; p.own = a.own; p.status = a.status;
    p.L = a.L; p.W = a.W; p.nwb = (a.L + a.W - 1) / a.W;
    p.NW = (int64_t)a.B * a.Hkv * p.nwb; p.cap = a.cap; p.Nc = a.L / a.S;
    p.H = a.H; p.Hkv = a.Hkv; p.topk = a.topk; p.S = a.S; p.add_own = a.own_chunk;
    p.lm_bf16 = a.lm_bf16;
    p.q3d = q3d ? 1 : 0;
    p.scale = a.scale;
    p.scale_log2e = a.scale * 1.4426950408889634f;
    kern<<<(unsigned)a.num_sms, kThreads, C::SMEM, st>>>(mq, mk, mv, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t rows = (int64_t)a.B * a.L * a.H;
    constexpr int kWarps = 8;
    fuse_kernel<D, G><<<(unsigned)((rows + kWarps - 1) / kWarps), 32 * kWarps, 0, st>>>(
        a.part, a.own, a.logits, a.idx, rows, a.H, a.Hkv, a.topk, a.w_out,
        (__nv_bfloat16 *)a.O);
    return cudaGetLastError();
}

int64_t attend_tc_max_windows() { return kMaxWindows; }

bool attend_tc_supported(bool bf16, int G, int d) {
    return bf16 && (G == 8 || G == 16) && (d == 64 || d == 128) && encode_fn() != nullptr;
}

cudaError_t launch_attend_tc(const TcLaunch &a, int d, cudaStream_t st) {
    const int G = a.H / a.Hkv;
    if (d == 128) return G == 8 ? launch_attend_tc_t<128, 8>(a, st) : launch_attend_tc_t<128, 16>(a, st);
    return G == 8 ? launch_attend_tc_t<64, 8>(a, st) : launch_attend_tc_t<64, 16>(a, st);
}

}  // namespace hsa
