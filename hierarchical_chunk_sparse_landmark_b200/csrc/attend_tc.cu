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
//   P = 2^-6 exp(S*scale - rowmax)          per row in registers, bf16 -> TMEM
//   O = P . V_chunk                         M=128, N=d, K=64  (tcgen05, A from TMEM)
//   partial[t, g, k] = O (fp16); per (t, h, k): the fusion logit
//   scale * (S[:,64] + S[:,65]) and f = 1 / sum of the row's P
//
// Own tiles: 128/G consecutive tokens of a chunk against that chunk with the
// causal mask (keys c*S .. t); their output (the own-chunk term, same scaling,
// f = own_chunk / row sum) goes to an fp16 array.  fuse_kernel then completes
// the method, one warp per (t, g):
//   w = softmax over the token's selected chunks of the logits,
//   O = f_own * own + sum_k w_k * f_k * partial_k  (bf16 out).
// Union-softmax variant (one softmax over the keys of all selected chunks and
// the own chunk; Dynamic Hierarchical Sparse Attention review): the tiles
// store each row's scaled maximum x = scale * max(S) and row sum r instead of
// (fusion logit, 1 / r), and the fusion is
//   O = sum_k e^{x_k - M} partial_k / sum_k e^{x_k - M} r_k,  M = max_k x_k
// over the selected chunks and the own chunk (when attended); both sums carry
// the same 2^-6, so it cancels.
//
// attend_tc_kernel: one persistent block per SM walks the tile queue (a flat
// list of tile descriptors) with these roles, linked by mbarriers, a ring of
// three Q/K shared-memory slots, a ring of three V slots and double-buffered
// TMEM accumulators (S, P and O); each role reads the descriptors (and its
// row's entry code) itself, one to two tiles ahead, into registers:
//   warps 0, 15  producers (even / odd tiles: TMA of the chunk's K, its
//                           landmark rows into key rows 64/65, the Q rows --
//                           one box per entry, its G query-head rows -- and V)
//   warp 1       MMA issuer for S
//   warp 14      MMA issuer for P.V
//   warps 2-9    softmax   (two groups taking alternate tiles; thread = tile
//                           row = TMEM lane)
//   warps 10-13  epilogue  (TMEM -> fp16 partial slots / own-chunk term)
// Tiles are independent, so no block waits on another.  Every wait is
// bounded; on expiry the block sets the status flag in the workspace, lets
// in-flight copies land, frees its TMEM and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "attend_tc.h"
#include "common.cuh"
#include "tc.cuh"
#include "tmap.cuh"

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
    static constexpr int K_TMA_BYTES = 64 * D * 2;   // the 64 key rows (rows 64+ are written in smem)
    // Q and K are dead once S is computed, V only after P.V: they live in
    // separate rings of three slots each, so loads run up to three tiles ahead.  Every slot is a multiple of 1 KB (128-byte swizzle atoms).
    static constexpr int NQK = 3, NVP = 3;
    static constexpr int QK_STAGE = Q_BYTES + K_BYTES;
    static constexpr int VP_STAGE = V_BYTES;
    static constexpr int BAR_OFF = NQK * QK_STAGE + NVP * VP_STAGE;
    static constexpr int BAR_BYTES = 512;        // mbarriers + TMEM address + abort flag
    static constexpr int SMEM = 1024 + BAR_OFF + BAR_BYTES;
    // TMEM: S[2] at columns 0 / 128 (80 used); P[2] (bf16 pairs, 32 columns)
    // right after each S at 80 / 208; O[2] at 256 / 256 + D
    static constexpr uint32_t S_COL = 128;
    static constexpr uint32_t P_OFF = 80;
    static constexpr uint32_t O_COL = 256;
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(QK_STAGE % 1024 == 0 && VP_STAGE % 1024 == 0, "slots must keep 1 KB alignment");
};

struct TcParams {
    const int4 *tiles;            // [qlen] tile descriptors in queue order
    const int64_t *qlen;
    const int32_t *entries;
    float *zf;                    // [B, L, H, topk] x (fusion logit, 1 / chunk row sum)
    float *own_f;                 // [B, L, H] add_own / own-chunk row sum (union: add_own * row sum)
    float *own_m;                 // [B, L, H] own-chunk scale * row max (union softmax only)
    __half *part;                 // [B*L*Hkv*topk entries][D/16][G][16] chunk outputs
    __half *own;                  // [B*L*Hkv rows (t, g)][D/16][G][16] own-chunk term
    unsigned *status;
    int64_t L, Nc;
    int H, Hkv, topk, S, add_own;
    uint64_t hkv_mul;             // floor(2^32 / Hkv) + 1: bg / Hkv = (bg * hkv_mul) >> 32
    int lm_rows;                  // landmark rows per chunk: 1 (bf16) or 2 (bf16 high, low of fp32)
    int q3d;                      // Q map is the 3-D (cols, rows, d-half) view
    int union_softmax;            // what the rows store for the fusion (see the file comment)
    Chunks ch;                    // chunks of S tokens or variable-length ones (<= 64 tokens)
    float scale, scale_log2e;
};

constexpr long long kWaitBudget = 4000000000LL;    // SM cycles (about 2 s)
constexpr int kThreads = 512;                       // 16 warps
constexpr int kEpiWarp0 = 10;                       // softmax groups: warps 2-5, 6-9; epilogue 10-13
constexpr int kEpiEnd = 14;                         // epilogue warps end here
constexpr int kPvWarp = 14;                         // issues the P.V products
constexpr int kProducer2 = 15;                      // second producer (odd tiles)
constexpr int kOwnTileFlag = 1 << 30;               // in a descriptor's .w (bucket.cu)

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}
// Two floats to a bf16 pair on the integer pipe: add half an ulp of bf16 to
// the fp32 bit pattern and keep the high halves (one byte permute).  Rounds to
// nearest with ties away from zero (round-to-nearest-even differs only on
// exact ties); used for P, whose pairs the P.V MMA reads from TMEM.
__device__ __forceinline__ uint32_t pack_bf16x2_int(float a, float b) {
    return __byte_perm(__float_as_uint(a) + 0x8000u, __float_as_uint(b) + 0x8000u, 0x7632);
}
// Chunk outputs are fp16 (11-bit significand): with bf16 the rounding of a
// partial and of the final O together could exceed the 2e-2 bf16 output
// tolerance where |O| approaches 4.
__device__ __forceinline__ uint32_t pack_f16x2(float a, float b) {
    __half2 v = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}
__device__ __forceinline__ float2 unpack_f16x2(uint32_t u) {
    return __half22float2(*reinterpret_cast<const __half2 *>(&u));
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
// Warp-level forms: every lane waits (a wait by one lane and a broadcast was
// slower) and the warp votes on the outcome, so a break on abort is
// warp-uniform; one arrive stands for all 32 lanes, each of which fenced its
// own prior tcgen05 work before the warp sync.
// Barriers that warps release count warps, not threads: a per-thread arrive
// is one shared-memory atomic each, and 640 of them per tile queued up
// behind every other barrier operation of the block.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort) {
    return __all_sync(0xffffffffu, wait_bar(bar, parity, abort)) != 0;
}
__device__ __forceinline__ void warp_arrive(uint64_t *bar) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) tc::mbar_arrive(bar);
}

// Parity to wait on before the u-th reuse of a ring slot (u >= 1): the
// consumer's release of use u-1.
__device__ __forceinline__ uint32_t reuse_parity(int64_t u) { return (uint32_t)((u + 1) & 1); }

// bg / Hkv by a multiply-high instead of a runtime divide (a long dependent
// sequence in every role's per-tile decode): exact while bg * Hkv < 2^32,
// which the host checks.
__device__ __forceinline__ int div_hkv(const TcParams &p, int64_t bg) {
    return (int)(((uint64_t)bg * p.hkv_mul) >> 32);
}

// A queue position decoded into one tile.
struct Tile {
    int64_t bg, first, t0;   // first entry (retrieved) or first token (own)
    int chunk, n, own;
};

__device__ __forceinline__ void decode_tile(const TcParams &p, const int4 &d, Tile &tl) {
    tl.bg = d.x;
    tl.own = (d.w & kOwnTileFlag) ? 1 : 0;
    tl.n = d.w & (kOwnTileFlag - 1);
    tl.chunk = d.y;                      // the tile's chunk (own tiles: the tokens' chunk)
    if (!tl.own) {
        tl.first = d.z; tl.t0 = 0;
    } else {
        tl.t0 = d.z; tl.first = 0;
    }
}

// Per-row view of a tile for the softmax and epilogue threads.
struct RowJob {
    Tile tl;
    int64_t t;
    int k, b, g;
    bool valid;
};

// Every role walks its own tiles j0, j0 + step, ... and reads their metadata
// itself: the descriptor two of its tiles ahead and this thread's entry code
// (row e) one tile ahead go into registers, so no role waits on a fresh load
// or on another role's hand-over.
struct TileFeed {
    int4 d1, d2;       // descriptors of the current and the next tile
    int32_t c1;        // this row's entry code in the current tile
};
__device__ __forceinline__ int4 load_desc(const TcParams &p, int64_t j, int64_t my_tiles) {
    return j < my_tiles ? __ldg(p.tiles + blockIdx.x + j * gridDim.x) : make_int4(0, 0, 0, 0);
}
__device__ __forceinline__ int32_t load_code(const TcParams &p, const int4 &d, int e) {
    Tile tl;
    decode_tile(p, d, tl);
    if (e >= tl.n) return 0;
    return tl.own ? (int32_t)((tl.t0 + e) * 32) : __ldg(p.entries + tl.first + e);
}
__device__ __forceinline__ void feed_init(TileFeed &f, const TcParams &p, int64_t j0, int64_t step,
                                          int64_t my_tiles, int e) {
    f.d1 = load_desc(p, j0, my_tiles);
    f.d2 = load_desc(p, j0 + step, my_tiles);
    f.c1 = load_code(p, f.d1, e);
}
// The row job of the current tile; advances the feed to the next one.
__device__ __forceinline__ RowJob feed_next(TileFeed &f, const TcParams &p, int64_t j, int64_t step,
                                            int64_t my_tiles, int e) {
    const int4 d3 = load_desc(p, j + 2 * step, my_tiles);
    const int32_t c2 = load_code(p, f.d2, e);
    RowJob rj;
    decode_tile(p, f.d1, rj.tl);
    rj.valid = e < rj.tl.n;
    rj.t = f.c1 >> 5;
    rj.k = f.c1 & 31;
    rj.b = div_hkv(p, rj.tl.bg);
    rj.g = (int)rj.tl.bg - rj.b * p.Hkv;
    f.d1 = f.d2; f.d2 = d3; f.c1 = c2;
    return rj;
}

template <int D, int G>
__global__ void __launch_bounds__(kThreads, 1)
attend_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmL,
                 const TcParams p) {
    using C = TcCfg<D, G>;
    grid_dep_wait();                      // the work lists are written by the previous kernels
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    // Q/K slot q: [Q | K;l]; V slot v
    auto sQ = [&](int q) { return smem + q * C::QK_STAGE; };
    auto sK = [&](int q) { return smem + q * C::QK_STAGE + C::Q_BYTES; };
    auto sV = [&](int v) { return smem + C::NQK * C::QK_STAGE + v * C::VP_STAGE; };
    uint64_t *bars = (uint64_t *)(smem + C::BAR_OFF);
    uint64_t *qk_full = bars, *qk_empty = bars + 3;                    // [NQK]
    uint64_t *v_full = bars + 6, *vp_empty = bars + 9;                 // [NVP]
    uint64_t *sfull = bars + 12, *sfree = bars + 14, *pfull = bars + 16;
    uint64_t *ofull = bars + 18, *ofree = bars + 20, *pempty = bars + 22;
    uint32_t *s_tmem = (uint32_t *)(bars + 24);
    static_assert(24 * 8 + 8 <= C::BAR_BYTES, "barrier block overflows its reserve");
    volatile int *s_abort = (volatile int *)(s_tmem + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // key rows 64..79 of every K block: the landmark rows land in 64 (and 65)
    // by TMA; the rest stay zero (row 65 too when landmarks are bf16)
    for (int i = tid; i < C::NQK * C::KB * 16 * 8; i += kThreads) {
        const int q = i / (C::KB * 128), kb = (i / 128) % C::KB, o = i % 128;
        reinterpret_cast<uint4 *>(sK(q) + kb * C::KBLK + 64 * 128)[o] = make_uint4(0u, 0u, 0u, 0u);
    }
    tc::fence_proxy_async_smem();
    if (warp == 1) {
        tc::tmem_alloc(s_tmem, C::TMEM_COLS);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        for (int q = 0; q < C::NQK; ++q) {
            tc::mbar_init(&qk_full[q], 1);     // producer: landmark rows written, Q/K loads expected
            tc::mbar_init(&qk_empty[q], 1);    // S MMA done
        }
        for (int v = 0; v < C::NVP; ++v) {
            tc::mbar_init(&v_full[v], 1);
            tc::mbar_init(&vp_empty[v], 1);    // P.V MMA done
        }
        for (int s = 0; s < 2; ++s) {
            tc::mbar_init(&sfull[s], 1);
            tc::mbar_init(&sfree[s], 4);       // one arrive per softmax warp
            tc::mbar_init(&pfull[s], 4);
            tc::mbar_init(&ofull[s], 1);
            tc::mbar_init(&ofree[s], 4);       // one arrive per epilogue warp
            tc::mbar_init(&pempty[s], 1);      // P.V done: TMEM P slot free
        }
        *s_abort = 0;
        tc::fence_barrier_init();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *s_tmem;
    const int64_t qlen = *p.qlen;
    const int64_t L = p.L;
    const int H = p.H, Hkv = p.Hkv, topk = p.topk;
    const int64_t my_tiles = qlen > blockIdx.x ? (qlen - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;

    if (warp == 0 || warp == kProducer2) {
        // ------------------------------------------------------------ producers
        // Producer pid takes the tiles j = 2u + pid.  The descriptor of tile
        // u + 2 and the entry codes of tile u + 1 are loaded into registers one
        // iteration ahead, so their latency hides behind the current tile.
        const int pid = warp == 0 ? 0 : 1;
        const int64_t my_u = (my_tiles - pid + 1) / 2;
        auto load_desc = [&](int64_t u) -> int4 {
            return u < my_u ? __ldg(p.tiles + blockIdx.x + (2 * u + pid) * gridDim.x) : make_int4(0, 0, 0, 0);
        };
        auto load_code = [&](const int4 &d) -> int32_t {
            Tile tl;
            decode_tile(p, d, tl);
            return (!tl.own && lane < tl.n) ? __ldg(p.entries + tl.first + lane) : 0;
        };
        // a window's query rows are re-read by every tile of their entries: keep
        // them in L2 ahead of the chunk outputs streaming out (those go evict-first)
        uint64_t pol_q;
        asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol_q));
        int4 d_cur = load_desc(0), d_nxt = load_desc(1);
        int32_t code_cur = load_code(d_cur);
        for (int64_t u = 0; u < my_u; ++u) {
            const int4 d_n2 = load_desc(u + 2);
            const int32_t code_nxt = load_code(d_nxt);
            const int64_t j = 2 * u + pid;
            Tile d0;
            decode_tile(p, d_cur, d0);
            const int32_t c0 = lane < d0.n ? (d0.own ? (int32_t)((d0.t0 + lane) * 32) : code_cur) : 0;
            const int bq = div_hkv(p, d0.bg);
            const int gq = (int)d0.bg - bq * Hkv;

            int ok = 1;
            // Q/K slot j % 3, free once the S of tile j - 3 is done: the chunk's
            // K rows, its landmark (bf16 high / low parts as key rows 64, 65)
            // and one Q box per entry (all G query-head rows, both halves of d
            // when the 3-D view is available), all on one transaction count
            const int q = (int)(j % C::NQK);
            if (lane == 0 && j >= C::NQK) ok = wait_bar(&qk_empty[q], reuse_parity(j / C::NQK), s_abort);
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            const int krow = (int)(d0.bg * L + chunk_first(p.ch, d0.chunk));
            if (lane == 0) {
                const uint32_t lbytes = d0.own ? 0u : (uint32_t)(C::KB * 128 * p.lm_rows);
                tc::mbar_expect_tx(&qk_full[q], (uint32_t)(d0.n * G * D * 2 + C::K_TMA_BYTES) + lbytes);
#pragma unroll
                for (int kb = 0; kb < C::KB; ++kb)
                    tc::tma_load_2d(sK(q) + kb * C::KBLK, &tmK, &qk_full[q], kb * 64, krow);
                if (!d0.own) {
                    const int lrow = (int)(d0.bg * p.Nc + d0.chunk);
#pragma unroll
                    for (int kb = 0; kb < C::KB; ++kb) {
                        if (p.lm_rows == 2)
                            tc::tma_load_3d(sK(q) + kb * C::KBLK + 64 * 128, &tmL, &qk_full[q], kb * 64, lrow, 0);
                        else
                            tc::tma_load_2d(sK(q) + kb * C::KBLK + 64 * 128, &tmL, &qk_full[q], kb * 64, lrow);
                    }
                }
            }
            __syncwarp();
            if (lane < d0.n) {
                const int qrow = (int)((bq * L + (int64_t)(c0 >> 5)) * H + (int64_t)gq * G);
                if (p.q3d) {
                    tc::tma_load_3d_hint(sQ(q) + lane * (C::KB * G * 128), &tmQ, &qk_full[q], 0, qrow, 0,
                                         pol_q);
                } else {
#pragma unroll
                    for (int kb = 0; kb < C::KB; ++kb)
                        tc::tma_load_2d_hint(sQ(q) + kb * (128 * 128) + lane * G * 128, &tmQ, &qk_full[q],
                                             kb * 64, qrow, pol_q);
                }
            }

            // V of the chunk into V slot j % 3, free once the P.V of tile j - 3
            // is done
            const int v = (int)(j % C::NVP);
            if (lane == 0) {
                if (j >= C::NVP) ok = wait_bar(&vp_empty[v], reuse_parity(j / C::NVP), s_abort);
                if (ok) {
                    tc::mbar_expect_tx(&v_full[v], (uint32_t)C::V_BYTES);
#pragma unroll
                    for (int kb = 0; kb < C::KB; ++kb)
                        tc::tma_load_2d(sV(v) + kb * 8192, &tmV, &v_full[v], kb * 64, krow);
                }
            }
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            d_cur = d_nxt; d_nxt = d_n2; code_cur = code_nxt;
        }
    } else if (warp == 1 || warp == kPvWarp) {
        // ------------------------------------------------------------ MMA issuers
        // Two threads issue tcgen05.mma: warp 1 the S products, warp 14 the
        // P.V products, each waiting only on its own inputs, so one stream's
        // barrier checks (each an mbarrier round trip of ~100+ cycles) never
        // delay the other.  The streams touch disjoint TMEM columns (S at
        // s*128 .. +80, P at s*128 + 80 .. +112, O at 256 + s*D) and commit to
        // their own barriers; a commit tracks only its own thread's MMAs.
        if (lane == 0) {
            constexpr uint32_t IDESC_S = tc::idesc_bf16_f32(128, C::NS, false);
            constexpr uint32_t IDESC_O = tc::idesc_bf16_f32(128, D, true);
            // Descriptors are built once for slot 0; a slot or a K step moves
            // only the start-address field (bytes / 16; every operand sits below
            // 256 KB, so the 14-bit field never carries), so an MMA costs the
            // issuing thread one add per operand.
            const uint64_t ad0 = p.q3d ? tc::sdesc_sw128(tc::smem_u32(sQ(0)), 16, C::KB * G * 128)
                                       : tc::sdesc_sw128(tc::smem_u32(sQ(0)), 16, 1024);
            const uint32_t a_kb = p.q3d ? (uint32_t)(G * 128 / 16) : (uint32_t)(16384 / 16);
            const uint64_t bd0 = tc::sdesc_sw128(tc::smem_u32(sK(0)), 16, 1024);
            const uint64_t vd0 = tc::sdesc_sw128(tc::smem_u32(sV(0)), 8192, 1024);
            auto issue_pv = [&](int64_t i) {
                const int s = (int)(i & 1), v = (int)(i % C::NVP);
                const uint64_t vd = vd0 + (uint64_t)(v * (C::VP_STAGE / 16));
                const uint32_t pa = tmem + s * C::S_COL + C::P_OFF, od = tmem + C::O_COL + s * D;
                tc::fence_after_sync();
                // A = P from TMEM: 16 keys = 8 packed columns per step
                tc::mma_bf16_ts(od, pa, vd, IDESC_O, 0u);
#pragma unroll
                for (int kk = 1; kk < 4; ++kk)
                    tc::mma_bf16_ts(od, pa + kk * 8, vd + (uint64_t)(kk * 2048 / 16), IDESC_O, 1u);
                tc::mma_commit(&ofull[s]);
                tc::mma_commit(&vp_empty[v]);
                tc::mma_commit(&pempty[s]);
            };
            auto issue_s = [&](int64_t j) {
                const int s = (int)(j & 1), q = (int)(j % C::NQK);
                const uint64_t ad = ad0 + (uint64_t)(q * (C::QK_STAGE / 16));
                const uint64_t bd = bd0 + (uint64_t)(q * (C::QK_STAGE / 16));
                const uint32_t sd = tmem + s * C::S_COL;
                tc::fence_after_sync();
#pragma unroll
                for (int kb = 0; kb < C::KB; ++kb)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc::mma_bf16(sd, ad + (uint64_t)(kb * a_kb + kk * 2),
                                     bd + (uint64_t)(kb * (C::KBLK / 16) + kk * 2), IDESC_S, (kb | kk) ? 1u : 0u);
                tc::mma_commit(&sfull[s]);
                tc::mma_commit(&qk_empty[q]);
            };
            if (warp == 1) {
                // S of tile j: its Q/K slot loaded, S slot j%2 read by the
                // softmax of tile j-2
                for (int64_t j = 0; j < my_tiles; ++j) {
                    if (!wait_bar(&qk_full[j % C::NQK], (uint32_t)((j / C::NQK) & 1), s_abort)) break;
                    if (j >= 2 && !wait_bar(&sfree[j & 1], reuse_parity(j >> 1), s_abort)) break;
                    issue_s(j);
                }
            } else {
                // P.V of tile i: P written, V loaded, O slot i%2 read by the
                // epilogue of tile i-2
                for (int64_t i = 0; i < my_tiles; ++i) {
                    if (!wait_bar(&pfull[i & 1], (uint32_t)((i >> 1) & 1), s_abort)) break;
                    if (!wait_bar(&v_full[i % C::NVP], (uint32_t)((i / C::NVP) & 1), s_abort)) break;
                    if (i >= 2 && !wait_bar(&ofree[i & 1], reuse_parity(i >> 1), s_abort)) break;
                    issue_pv(i);
                }
            }
        }
    } else if (warp < kEpiWarp0) {
        // ------------------------------------------------------------ softmax
        const int q4 = warp & 3;                  // TMEM lane quarter
        const int r = q4 * 32 + lane;             // tile row
        const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
        const int e = r / G, h = r % G;
        const int sg = (warp - 2) >> 2;
        TileFeed feed;
        feed_init(feed, p, sg, 2, my_tiles, e);
        for (int64_t j = sg; j < my_tiles; j += 2) {
            const RowJob cur = feed_next(feed, p, j, 2, my_tiles, e);
            const int s = (int)(j & 1);
            const int64_t b = cur.b;
            const int g = cur.g;
            if (!warp_wait(&sfull[s], (uint32_t)((j >> 1) & 1), s_abort)) break;
            tc::fence_after_sync();
            float s0[32], s1[32], l_hi, l_lo;
            const uint32_t ta = tmem + s * C::S_COL + lane_off;
            tc::tmem_ld32(ta, s0);
            tc::tmem_ld32(ta + 32, s1);
            tc::tmem_ld2(ta + 64, l_hi, l_lo);
            tc::tmem_wait_ld();
            tc::fence_before_sync();
            warp_arrive(&sfree[s]);
            // own-chunk rows see the keys of their chunk up to t only, and a
            // variable-length chunk has fewer than 64 keys (the rows past it
            // belong to the next chunk): mask the rest to -inf
            int nk = 64;
            if (cur.tl.own)
                nk = cur.valid ? (int)(cur.t - chunk_first(p.ch, cur.tl.chunk)) + 1 : 64;
            else if (p.ch.bounds)
                nk = chunk_len(p.ch, cur.tl.chunk);
            if (nk < 64) {
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    if (c >= nk) s0[c] = -INFINITY;
                    if (c + 32 >= nk) s1[c] = -INFINITY;
                }
            }
            float m4[4] = {s0[0], s0[1], s1[0], s1[1]};
#pragma unroll
            for (int c = 2; c < 32; c += 2) {
                m4[0] = tc::max3(m4[0], s0[c], s0[c + 1]);
                m4[1] = tc::max3(m4[1], s1[c], s1[c + 1]);
            }
            const float mx = fmaxf(fmaxf(m4[0], m4[2]), fmaxf(m4[1], m4[3]));
            // P = exp(S*scale - rowmax), unnormalised (1/rowsum is applied by
            // fuse_kernel; the 2^-6, an exponent shift, keeps P.V within
            // max |V| for its fp16 store)
            const float ms = fmaf(mx, p.scale_log2e, 6.f);
            const uint64_t c2 = pack_f2(p.scale_log2e, p.scale_log2e), m2 = pack_f2(-ms, -ms);
            uint64_t l2 = 0ull;
#pragma unroll
            for (int c = 0; c < 32; c += 2) {
                float a0, a1, b0, b1;
                unpack_f2(ffma2(pack_f2(s0[c], s0[c + 1]), c2, m2), a0, a1);
                unpack_f2(ffma2(pack_f2(s1[c], s1[c + 1]), c2, m2), b0, b1);
                s0[c] = tc::ex2_approx(a0); s0[c + 1] = tc::ex2_approx(a1);
                s1[c] = tc::ex2_approx(b0); s1[c + 1] = tc::ex2_approx(b1);
                l2 = add_f2(l2, add_f2(pack_f2(s0[c], s0[c + 1]), pack_f2(s1[c], s1[c + 1])));
            }
            if (cur.valid) {
                const int64_t hrow = (b * L + cur.t) * H + (int64_t)g * G + h;
                const float rs = sum_f2(l2);
                if (!p.union_softmax) {
                    const float f = __fdividef(cur.tl.own ? (float)p.add_own : 1.f, rs);
                    if (cur.tl.own)
                        p.own_f[hrow] = f;
                    else
                        reinterpret_cast<float2 *>(p.zf)[hrow * topk + cur.k] =
                            make_float2(p.scale * (l_hi + l_lo), f);
                } else if (cur.tl.own) {
                    p.own_f[hrow] = (float)p.add_own * rs;
                    p.own_m[hrow] = p.scale * mx;
                } else {
                    reinterpret_cast<float2 *>(p.zf)[hrow * topk + cur.k] = make_float2(p.scale * mx, rs);
                }
            }
            // P goes into TMEM next to S slot s (this thread's lane, keys packed
            // in pairs), free once the P.V of tile j - 2 is done
            uint32_t pk[32];
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                pk[c] = pack_bf16x2_int(s0[2 * c], s0[2 * c + 1]);
                pk[16 + c] = pack_bf16x2_int(s1[2 * c], s1[2 * c + 1]);
            }
            if (j >= 2 && !warp_wait(&pempty[s], reuse_parity(j >> 1), s_abort)) break;
            tc::tmem_st32(tmem + s * C::S_COL + C::P_OFF + lane_off, pk);
            tc::tmem_wait_st();
            tc::fence_before_sync();
            warp_arrive(&pfull[s]);
        }
    } else if (warp < kEpiEnd) {
        // ------------------------------------------------------------ epilogue
        const int q4 = warp & 3;
        const int r = q4 * 32 + lane;
        const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
        const int e = r / G, h = r % G;
        constexpr int NCH = D / 32;               // 32-column chunks of a row
        // chunk outputs are evicted from L2 first: the Q / K / V rows the
        // other tiles re-read stay (measured: 4 us of 160 on the train shape)
        uint64_t pol;
        asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
        TileFeed feed;
        feed_init(feed, p, 0, 1, my_tiles, e);
        for (int64_t j = 0; j < my_tiles; ++j) {
            const RowJob cur = feed_next(feed, p, j, 1, my_tiles, e);
            const int s = (int)(j & 1);
            const int64_t b = cur.b;
            const int g = cur.g;
            // one contiguous G*D block per (t, g, k) (own term: per (t, g)), 32-byte
            // pieces ordered [d/16][head]: the G heads' pieces of a column group
            // are adjacent, so every 256-bit store instruction writes whole lines
            const int64_t row = (b * L + cur.t) * Hkv + g;
            uint4 *blk = reinterpret_cast<uint4 *>(cur.tl.own ? p.own + row * (G * D)
                                                              : p.part + (row * topk + cur.k) * (G * D));
            if (!warp_wait(&ofull[s], (uint32_t)((j >> 1) & 1), s_abort)) break;
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
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        uint32_t w8[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) w8[i] = pack_f16x2(o[u][16 * hh + 2 * i], o[u][16 * hh + 2 * i + 1]);
                        uint32_t *dst = reinterpret_cast<uint32_t *>(blk) + ((((ch + u) * 2 + hh) * G + h) * 8);
                        asm volatile("st.global.L2::cache_hint.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8}, %9;"
                                     :: "l"(dst), "r"(w8[0]), "r"(w8[1]), "r"(w8[2]), "r"(w8[3]), "r"(w8[4]),
                                        "r"(w8[5]), "r"(w8[6]), "r"(w8[7]), "l"(pol) : "memory");
                    }
                }
            }
            tc::fence_before_sync();
            warp_arrive(&ofree[s]);
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
// One warp per (t, g): w = softmax over the token's selected chunks of the
// logits (per head), O = f_own * own + sum_k w_k * f_k * partial_k, f = the
// reciprocal row sums of the unnormalised chunk outputs.  A slot's partials
// of the whole group are one contiguous block of 32-byte pieces ordered
// [d/16][G] (G*d*2 bytes; the own term has the same layout), read with
// coalesced 16-byte loads: lane l takes 16-byte pieces l + 32 i (halves of the
// 32-byte pieces), all of head (l / 2) % G (G divides 16), columns
// 16 * ((l + 32 i) / 2G) + 8 * (l % 2) .. +8.  The own term's and
// the first slots' loads go out before the selection count is known.
// Two blocks per SM where a lane's pieces allow (G*d <= 1024), else one: the
// loads in flight per warp, not the warp count, keep HBM busy.
template <int D, int G, int KP>
__global__ void __launch_bounds__(256, (G * D / 256) <= 4 ? 2 : 1)
fuse_kernel(const __half *__restrict__ part, const __half *__restrict__ own,
            const float2 *__restrict__ zf, const float *__restrict__ own_f,
            const float *__restrict__ own_m, int union_softmax,
            const int32_t *__restrict__ idx, int64_t groups, int H, int Hkv, int topk,
            float *__restrict__ w_out, __nv_bfloat16 *__restrict__ O) {
    constexpr int NP = G * D / 256;                  // 16-byte pieces per lane and slot
    constexpr int SLOT = G * D / 8;                  // 16-byte pieces per slot
    static_assert(NP >= 1 && 32 % G == 0, "a lane's pieces must all belong to one head");
    constexpr int SG = NP <= 4 ? 4 : 2;              // slots whose loads are in flight together
    static_assert(KP % SG == 0 && KP <= 32, "slots are taken SG at a time");
    grid_dep_wait();                                 // the chunk outputs come from attend_tc_kernel
    const int lane = threadIdx.x & 31;
    // Rows in reverse: attend_tc_kernel writes the chunk outputs window by
    // window, so when it ends L2 still holds the last windows' outputs; those
    // are read first.  Every consumed 128-byte line is then discarded from L2
    // (the data is dead), so dirty lines still there are never written back.
    const int64_t lin = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    if (lin >= groups) return;
    const int64_t srow = groups - 1 - lin;           // srow = (b*L + t)*Hkv + g
    const int64_t bt = srow / Hkv;
    const int g = (int)(srow % Hkv);
    const int h = (lane >> 1) % G;
    const int64_t hrow = bt * H + (int64_t)g * G + h;
    const uint4 *pb = reinterpret_cast<const uint4 *>(part + srow * topk * (int64_t)(G * D));
    const uint4 *ob = reinterpret_cast<const uint4 *>(own + srow * (int64_t)(G * D));
    // The loads that do not depend on the selection go out first: the own term
    // and the first SG slots (a slot past the valid ones is zeroed below).
    uint4 rown[NP], raw[SG][NP];
#pragma unroll
    for (int i = 0; i < NP; ++i) rown[i] = ob[lane + 32 * i];
#pragma unroll
    for (int u = 0; u < SG; ++u)
#pragma unroll
        for (int i = 0; i < NP; ++i)
            raw[u][i] = u < topk ? pb[(int64_t)u * SLOT + lane + 32 * i] : make_uint4(0u, 0u, 0u, 0u);
    const int nsel = __popc(__ballot_sync(0xffffffffu, lane < topk && idx[srow * topk + lane] >= 0));
    // fusion weights of this lane's head: softmax of the logits over the valid slots
    // (union softmax: e^{x_k - M} over the slots and the own term, normalised by
    // the matching sum of row sums)
    const float2 *zh = zf + hrow * topk;
    float zx[KP];
#pragma unroll
    for (int k = 0; k < KP; ++k) zx[k] = k < nsel ? zh[k].x : -INFINITY;
    const float fown = own_f[hrow];
    const float xown = union_softmax && fown > 0.f ? own_m[hrow] : -INFINITY;
    float m = xown;
#pragma unroll
    for (int k = 0; k < KP; ++k) m = fmaxf(m, zx[k]);
    float den = union_softmax && fown > 0.f ? __expf(xown - m) * fown : 0.f;
#pragma unroll
    for (int k = 0; k < KP; ++k)
        den += k < nsel ? __expf(zx[k] - m) * (union_softmax ? zh[k].y : 1.f) : 0.f;
    const float inv = den > 0.f ? 1.f / den : 0.f;
    if (w_out && lane < 2 * G && (lane & 1) == 0)
        for (int k = 0; k < topk; ++k)
            w_out[hrow * topk + k] = (k < nsel && !union_softmax) ? __expf(zh[k].x - m) * inv : 0.f;
    float acc[NP][8];
    const float fo = union_softmax ? (fown > 0.f ? __expf(xown - m) * inv : 0.f) : fown;
    constexpr int LINES = G * D * 2 / 128;           // 128-byte lines of one slot
#pragma unroll
    for (int i = 0; i < NP; ++i) {
        const uint32_t *w2 = reinterpret_cast<const uint32_t *>(&rown[i]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = unpack_f16x2(w2[e]);
            acc[i][2 * e] = fo * f.x;
            acc[i][2 * e + 1] = fo * f.y;
        }
    }
    __syncwarp();
    for (int l = lane; l < LINES; l += 32) tc::discard_l2(reinterpret_cast<const uint8_t *>(ob) + l * 128);
#pragma unroll
    for (int k0 = 0; k0 < KP; k0 += SG) {
        if (k0 >= nsel) break;
        if (k0 > 0) {
#pragma unroll
            for (int u = 0; u < SG; ++u)
#pragma unroll
                for (int i = 0; i < NP; ++i)
                    raw[u][i] = k0 + u < nsel ? pb[(int64_t)(k0 + u) * SLOT + lane + 32 * i]
                                              : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < SG; ++u) {
            const bool valid = k0 + u < nsel;
            const float wk = !valid ? 0.f
                             : union_softmax ? __expf(zx[k0 + u] - m) * inv
                                             : __expf(zx[k0 + u] - m) * inv * zh[k0 + u].y;
#pragma unroll
            for (int i = 0; i < NP; ++i) {
                const uint4 rv = valid ? raw[u][i] : make_uint4(0u, 0u, 0u, 0u);
                const uint32_t *w2 = reinterpret_cast<const uint32_t *>(&rv);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = unpack_f16x2(w2[e]);
                    acc[i][2 * e] = fmaf(wk, f.x, acc[i][2 * e]);
                    acc[i][2 * e + 1] = fmaf(wk, f.y, acc[i][2 * e + 1]);
                }
            }
        }
        __syncwarp();
        const int nv = nsel - k0 < SG ? nsel - k0 : SG;  // slots of this group that were read
        for (int l = lane; l < nv * LINES; l += 32)
            tc::discard_l2(reinterpret_cast<const uint8_t *>(pb + (int64_t)k0 * SLOT) + l * 128);
    }
#pragma unroll
    for (int i = 0; i < NP; ++i) {
        const int pc = lane + 32 * i;
        const int c8 = (pc >> 1) / G * 2 + (pc & 1);
        *reinterpret_cast<uint4 *>(O + hrow * D + c8 * 8) =
            make_uint4(pack_bf16x2(acc[i][0], acc[i][1]), pack_bf16x2(acc[i][2], acc[i][3]),
                       pack_bf16x2(acc[i][4], acc[i][5]), pack_bf16x2(acc[i][6], acc[i][7]));
    }
}

// ---------------------------------------------------------------- host side
template <int D, int G>
static cudaError_t launch_attend_tc_t(const TcLaunch &a, cudaStream_t st, cudaEvent_t mid) {
    using C = TcCfg<D, G>;
    CUtensorMap mq, mk, mv, ml;
    // the single-box entry layout has a uniform 8-row atom stride only when an
    // entry is exactly one atom (G = 8) and d has two halves
    bool q3d = (G == 8 && D == 128) &&
               make_map_q3d(&mq, a.Q, (uint64_t)a.B * a.L * a.H, D, G);
    if (!q3d && !make_map(&mq, a.Q, (uint64_t)a.B * a.L * a.H, D, G)) return cudaErrorInvalidValue;
    if (!make_map(&mk, a.K, (uint64_t)a.B * a.Hkv * a.L, D, 64) ||
        !make_map(&mv, a.V, (uint64_t)a.B * a.Hkv * a.L, D, 64))
        return cudaErrorInvalidValue;
    const uint64_t lrows = (uint64_t)a.B * a.Hkv * a.Nc;
    if (lrows == 0) ml = mk;                       // no chunk tiles: the map is never used
    else if (!(a.lm_bf16 ? make_map(&ml, a.lm, lrows, D, 1) : make_map_planes(&ml, a.lm, lrows, D)))
        return cudaErrorInvalidValue;
    auto kern = attend_tc_kernel<D, G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    TcParams p;
    p.tiles = a.tiles; p.qlen = a.qlen;
    p.entries = a.entries; p.zf = a.zf; p.own_f = a.own_f; p.own_m = a.own_m;
    p.union_softmax = a.union_softmax;
    p.ch.bounds = a.bounds; p.ch.tok_chunk = a.tok_chunk; p.ch.L = a.L; p.ch.S = a.S;
    p.part = a.part; p.own = a.own; p.status = a.status;
    p.L = a.L; p.Nc = a.Nc;
    p.H = a.H; p.Hkv = a.Hkv; p.topk = a.topk; p.S = a.S; p.add_own = a.own_chunk;
    p.hkv_mul = (uint64_t)(0x100000000ull / (uint64_t)a.Hkv) + 1ull;
    p.lm_rows = a.lm_bf16 ? 1 : 2;
    p.q3d = q3d ? 1 : 0;
    p.scale = a.scale;
    p.scale_log2e = a.scale * 1.4426950408889634f;
    e = launch_pdl(kern, dim3((unsigned)a.num_sms), dim3(kThreads), (size_t)C::SMEM, st, mq, mk, mv, ml, p);
    if (e != cudaSuccess) return e;
    // with a timing event between the two kernels the fusion kernel is launched
    // plainly (an event between them ends the programmatic overlap anyway)
    if (mid && (e = cudaEventRecord(mid, st)) != cudaSuccess) return e;
    const int64_t groups = (int64_t)a.B * a.L * a.Hkv;
    constexpr int kWarps = 8;
    const dim3 fgrid((unsigned)((groups + kWarps - 1) / kWarps));
    auto fk = a.topk <= 8 ? fuse_kernel<D, G, 8> : a.topk <= 16 ? fuse_kernel<D, G, 16> : fuse_kernel<D, G, 32>;
    return launch_pdl(fk, fgrid, dim3(32 * kWarps), 0, st, a.part, a.own,
                      (const float2 *)a.zf, (const float *)a.own_f, (const float *)a.own_m,
                      a.union_softmax, (const int32_t *)a.idx, groups,
                      a.H, a.Hkv, a.topk, a.w_out, (__nv_bfloat16 *)a.O);
}

// The work lists hold no per-window state in shared memory any more; the
// window count only sizes device arrays.
int64_t attend_tc_max_windows() { return int64_t(1) << 20; }

bool attend_tc_supported(bool bf16, int G, int d) {
    return bf16 && (G == 8 || G == 16) && (d == 64 || d == 128) && encode_fn() != nullptr;
}

// `mid` (may be null) is recorded between the attention and fusion kernels.
cudaError_t launch_attend_tc(const TcLaunch &a, int d, cudaStream_t st, cudaEvent_t mid) {
    const int G = a.H / a.Hkv;
    if (d == 128)
        return G == 8 ? launch_attend_tc_t<128, 8>(a, st, mid) : launch_attend_tc_t<128, 16>(a, st, mid);
    return G == 8 ? launch_attend_tc_t<64, 8>(a, st, mid) : launch_attend_tc_t<64, 16>(a, st, mid);
}

}  // namespace hsa
