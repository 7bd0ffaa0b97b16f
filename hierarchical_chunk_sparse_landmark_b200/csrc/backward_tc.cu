// backward_tc.cu -- the prefill backward on the 5th-generation tensor cores
// (bf16 inputs, G = 8 query heads per KV group, d = 128).
//
// Same gradients as backward.cu (HiLS Attention abstract: the retrieval scores
// are learned end to end; the selection is held fixed), organised around the
// forward's chunk tiles: a tile is one chunk's 64 keys/values and up to 16
// entries (token, slot) that selected it, 8 query-head rows each, so 128 rows.
// Per tile, with w the row's fusion weight (1 for the own chunk):
//
//   S  = Q.K^T, U = dO.V^T            M = 128 rows, N = 64 keys, K = d   (TMEM)
//   p  = softmax_j(scale S) (causal mask on own tiles), dw = sum_j p_j U_j
//   dS = scale w p (U - dw), wP = w p   (bf16, written to shared memory)
//   dV^T += dO^T . wP,  dK^T += Q^T . dS  M = d, N = 64, K = 128 rows (TMEM,
//                                         accumulated over the segment's tiles)
//   dQp  = dS . K                       M = 128 rows, N = d, K = 64 keys
//
// The transposed products read the Q / dO / K tiles already in shared memory
// as MN-major operands (no copy).  One persistent block per SM (8 compute
// warps, the two threads of a tile row -- one TMEM lane -- taking keys 0-31
// and 32-63, and an issuer warp for the MMAs and row loads; see the kernel)
// walks the segments of the chunks' sorted entry lists (at most 8 tiles each)
// and the own chunks (at most 4 tiles of 16 tokens); K and V are loaded once
// per segment.  dw and the dQ partial rows of every (row, slot) go to global
// memory; bwd_rowfin_kernel then forms dz = w (dw - sum w dw), sums the dQ
// partials and adds scale sum dz l; bwd_dl_kernel forms each segment's
// landmark gradient scale sum dz q; the ordered reduction of backward.cu adds
// the segments.  All in a fixed order: bit-reproducible.
//
// Precision: P and dS enter the second products as bf16 (as P does in the
// forward), so gradients carry ~2^-9 relative rounding per term.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "tc.cuh"
#include "tmap.cuh"

namespace hsa {

namespace {

constexpr int kBtThreads = 288;            // 8 compute warps (two threads per tile row:
                                           // keys 0-31, 32-63) and an issuer warp
constexpr long long kBtWait = 4000000000LL;       // SM cycles (about 2 s)
constexpr int BT_D = 128, BT_G = 8, BT_EPT = 16;  // d, heads per entry, entries per tile
// shared memory, offsets from a 1024-byte aligned base: two buffers of the
// tile's Q and dO rows, so the next tile's rows load during this tile's work
constexpr int QBUF = 32768;                // [16 entries][2 halves of d][8 rows][128 B]
constexpr int OFF_Q = 0;                   // Q[2]
constexpr int OFF_DO = OFF_Q + 2 * QBUF;   // dO[2]
constexpr int OFF_K = OFF_DO + 2 * QBUF;   // [2 halves][64 keys][128 B]
constexpr int OFF_V = OFF_K + 16384;
constexpr int OFF_DS = OFF_V + 16384;      // [128 rows][64 keys] bf16, 128B-swizzled
constexpr int OFF_WP = OFF_DS + 16384;
constexpr int OFF_RED = OFF_WP + 16384;    // [3][2 halves][128 rows] fp32: row max, sums
constexpr int OFF_BAR = OFF_RED + 3 * 2 * 128 * 4;   // mbarriers, TMEM address, abort flag
constexpr int BT_SMEM = 1024 + OFF_BAR + 128;
// TMEM columns (fp32): S and U twice (the next tile's products run during this
// tile's epilogue), the dQ partial, and the segment's dV^T and dK^T
constexpr uint32_t COL_SU = 0;             // buffer i: S at 128 i, U at 128 i + 64
constexpr uint32_t COL_DQ = 256, COL_DV = 384, COL_DK = 448;
constexpr uint32_t BT_TMEM_COLS = 512;

struct BtParams {
    const int4 *segs;
    const int32_t *nseg;
    const int32_t *entries;
    const float2 *coef;      // [B*L*H][topk]: .x = w (written by bwd_coefw_kernel)
    float *dw;               // [B*L*H][topk+1]: dw of every (row, slot); slot topk = own
    __half *dqp;             // [B*L*Hkv][topk+1][G][D]: dQ partial rows (fp16)
    float *part;             // per segment: dK [64][D], dV [64][D], dl [D]
    unsigned *status;
    int64_t L, NcAll;
    int H, Hkv, topk, S;
    float scale;
};

__device__ __forceinline__ bool bt_wait(uint64_t *bar, uint32_t parity, volatile int *abort) {
    if (tc::mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!tc::mbar_try_wait(bar, parity)) {
        if (*abort || clock64() - t0 > kBtWait) {
            *abort = 1;
            return false;
        }
    }
    return true;
}

__device__ __forceinline__ uint32_t pack2_bf16(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}

}  // namespace

// A tile's row of this thread: entry e = (tid % 128) / 8 of the tile, head
// h = tid % 8; threads tid and tid + 128 share the row (keys 0-31 and 32-63).
struct BtRow {
    int64_t t;
    int slot;
    bool valid;
};

// One segment: chunk c of (b, g), its entries (or its own tokens) in tiles of
// BT_EPT.
struct BtSeg {
    int64_t bg, b, c, first;
    int g, own, n_units, ntiles;
    int32_t ebase;
};
__device__ __forceinline__ BtSeg bt_segment(const BtParams &p, int64_t sidx) {
    const int4 sg = p.segs[sidx];
    BtSeg s;
    const int64_t q = sg.x;
    s.bg = q / p.NcAll;
    s.c = q % p.NcAll;
    s.b = s.bg / p.Hkv;
    s.g = (int)(s.bg % p.Hkv);
    s.own = sg.w;
    s.first = s.c * p.S;
    const int nkc = (int)(p.L - s.first < p.S ? p.L - s.first : p.S);
    s.n_units = s.own ? nkc : sg.z;      // tokens (own) or entries of the segment
    s.ntiles = (s.n_units + BT_EPT - 1) / BT_EPT;
    s.ebase = sg.y;
    return s;
}

// Barrier 1 over the eight compute warps (the issuer warp is not in it), with
// the AND of the threads' votes, so that a timeout is seen by all of them.
__device__ __forceinline__ bool cbar_and(bool v) {
    uint32_t r;
    asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
                 "bar.red.and.pred q, 1, 256, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
                 : "=r"(r) : "r"((uint32_t)v) : "memory");
    return r != 0;
}
__device__ __forceinline__ void cbar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// Roles: warps 0-7 compute (two threads per tile row: softmax, dS and w P,
// the dQ partial epilogue, the segment's dK / dV readout); warp 8 issues
// (lane 0 the MMAs, lanes 0-15 the row loads of their entries).  Per tile
// the issuer runs S and U of the next tile on the tensor pipe while the
// compute warps take this tile's softmax, then this tile's dV^T, dK^T and dQ
// products once the softmax has written dS and w P; the compute warps meet it
// only at the mbarriers below.
//   su_bar[buf]  S, U of a tile complete          (issuer -> compute)
//   ds_full      dS, w P of a tile written        (compute, one arrive per warp -> issuer)
//   o_bar        dV^T, dK^T, dQ of a tile done    (issuer -> both)
//   seg_free     dK^T / dV^T of a segment read    (compute, per warp -> issuer)
constexpr int kBtCompute = 256;
constexpr int kBtIssuer = 8;               // warp index of the issuer

__global__ void __launch_bounds__(kBtThreads, 1)
bwd_key_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
                  const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const BtParams p) {
    constexpr int D = BT_D, G = BT_G;
    const int64_t nseg = *p.nseg;
    if ((int64_t)blockIdx.x >= nseg) return;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t *bars = (uint64_t *)(sm + OFF_BAR);
    uint64_t *kv_bar = bars, *tma_bar = bars + 1, *su_bar = bars + 3, *o_bar = bars + 5;
    uint64_t *ds_full = bars + 6, *seg_free = bars + 7;
    uint32_t *s_tmem = (uint32_t *)(bars + 8);
    volatile int *s_abort = (volatile int *)(s_tmem + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t L = p.L;
    const int H = p.H, topk = p.topk;

    // rows of entries a tile does not fill are read by the transposed
    // products (times zero): they must hold finite values
    for (int i = tid; i < 4 * QBUF / 16; i += kBtThreads)
        reinterpret_cast<uint4 *>(sm + OFF_Q)[i] = make_uint4(0u, 0u, 0u, 0u);
    tc::fence_proxy_async_smem();
    if (warp == 0) {
        tc::tmem_alloc(s_tmem, BT_TMEM_COLS);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < 6; ++i) tc::mbar_init(&bars[i], 1);
        tc::mbar_init(ds_full, kBtCompute / 32);
        tc::mbar_init(seg_free, kBtCompute / 32);
        *s_abort = 0;
        tc::fence_barrier_init();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *s_tmem;
    bool ok = true;

    if (warp == kBtIssuer) {
        // ------------------------------------------------------------ issuer
        const uint32_t IDESC_SU = tc::idesc_bf16_f32(128, 64, false, false);
        const uint32_t IDESC_T = tc::idesc_bf16_f32(128, 64, true, true);     // M = d, N = keys
        const uint32_t IDESC_DQ = tc::idesc_bf16_f32(128, D, true, false);    // B = K, MN-major
        // descriptors of the fixed tiles (bytes >> 4 in the start field; a K step moves the start)
        const uint64_t bK = tc::sdesc_sw128(tc::smem_u32(sm + OFF_K), 16, 1024);     // keys x d
        const uint64_t bV = tc::sdesc_sw128(tc::smem_u32(sm + OFF_V), 16, 1024);
        const uint64_t bDS = tc::sdesc_sw128(tc::smem_u32(sm + OFF_DS), 16384, 1024);  // (keys, rows)
        const uint64_t bWP = tc::sdesc_sw128(tc::smem_u32(sm + OFF_WP), 16384, 1024);
        const uint64_t aDS = tc::sdesc_sw128(tc::smem_u32(sm + OFF_DS), 16, 1024);     // rows x keys
        const uint64_t bKt = tc::sdesc_sw128(tc::smem_u32(sm + OFF_K), 8192, 1024);    // (d, keys)
        uint32_t pkv = 0u, ptma[2] = {0u, 0u}, pds = 0u, po = 0u, pfree = 0u;
        bool dkdv_held = false;          // the compute warps still have to read a segment's dK / dV
        for (int64_t sidx = blockIdx.x; sidx < nseg && ok; sidx += gridDim.x) {
            const BtSeg sg = bt_segment(p, sidx);
            // Q / dO rows of tile ti into buffer ti % 2 (one 3-D box per entry:
            // its 8 head rows, both halves of d); the buffer's readers are done
            auto load_rows = [&](int ti) {
                const int buf = ti & 1;
                const int nvalid = sg.n_units - ti * BT_EPT < BT_EPT ? sg.n_units - ti * BT_EPT : BT_EPT;
                if (lane == 0) tc::mbar_expect_tx(&tma_bar[buf], (uint32_t)nvalid * 2u * 2048u);
                __syncwarp();
                if (lane < nvalid) {
                    const int u = ti * BT_EPT + lane;
                    const int64_t t = sg.own ? sg.first + u : (int64_t)(p.entries[sg.ebase + u] >> 5);
                    const int qrow = (int)((sg.b * L + t) * H + (int64_t)sg.g * G);
                    tc::tma_load_3d(sm + OFF_Q + buf * QBUF + lane * 2048, &tmQ, &tma_bar[buf], 0, qrow, 0);
                    tc::tma_load_3d(sm + OFF_DO + buf * QBUF + lane * 2048, &tmO, &tma_bar[buf], 0, qrow, 0);
                }
            };
            // S = Q.K^T and U = dO.V^T of tile ti
            auto issue_su = [&](int ti) {
                const int buf = ti & 1;
                const uint64_t aQ = tc::sdesc_sw128(tc::smem_u32(sm + OFF_Q + buf * QBUF), 16, 2048);
                const uint64_t aO = tc::sdesc_sw128(tc::smem_u32(sm + OFF_DO + buf * QBUF), 16, 2048);
                const uint32_t ds = tmem + COL_SU + 128u * (uint32_t)buf;
                tc::fence_after_sync();
#pragma unroll
                for (int kb = 0; kb < 2; ++kb)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint32_t acc = (kb | kk) ? 1u : 0u;
                        tc::mma_bf16(ds, aQ + (uint64_t)((kb * 1024 + kk * 32) >> 4),
                                     bK + (uint64_t)((kb * 8192 + kk * 32) >> 4), IDESC_SU, acc);
                        tc::mma_bf16(ds + 64, aO + (uint64_t)((kb * 1024 + kk * 32) >> 4),
                                     bV + (uint64_t)((kb * 8192 + kk * 32) >> 4), IDESC_SU, acc);
                    }
                tc::mma_commit(&su_bar[buf]);
            };
            // K and V of the chunk (every product of the previous segment is
            // complete: its last o_bar was waited below) and the first rows
            const int krow = (int)(sg.bg * L + sg.first);
            if (lane == 0) {
                tc::mbar_expect_tx(kv_bar, 2u * 16384u);
#pragma unroll
                for (int kb = 0; kb < 2; ++kb) {
                    tc::tma_load_2d(sm + OFF_K + kb * 8192, &tmK, kv_bar, kb * 64, krow);
                    tc::tma_load_2d(sm + OFF_V + kb * 8192, &tmV, kv_bar, kb * 64, krow);
                }
            }
            if (sg.ntiles > 0) load_rows(0);
            if (sg.ntiles > 1) load_rows(1);
            ok = bt_wait(kv_bar, pkv, s_abort) && (sg.ntiles == 0 || bt_wait(&tma_bar[0], ptma[0], s_abort));
            ok = __all_sync(0xffffffffu, ok);
            pkv ^= 1u;
            if (sg.ntiles > 0) ptma[0] ^= 1u;
            if (!ok) break;
            if (sg.ntiles > 0 && lane == 0) issue_su(0);
            for (int ti = 0; ti < sg.ntiles; ++ti) {
                const int buf = ti & 1, nb = buf ^ 1;
                // the segment's first dV^T / dK^T products overwrite the
                // accumulators of the previous one: its readout must be done
                if (ti == 0 && dkdv_held) {
                    if (!__all_sync(0xffffffffu, bt_wait(seg_free, pfree, s_abort))) { ok = false; break; }
                    pfree ^= 1u;
                    dkdv_held = false;
                }
                if (!__all_sync(0xffffffffu, bt_wait(ds_full, pds, s_abort))) { ok = false; break; }
                pds ^= 1u;
                // dV^T += dO^T . wP, dK^T += Q^T . dS (over the tile's 128 rows), dQp = dS . K
                if (lane == 0) {
                    tc::fence_after_sync();
                    const uint64_t tQ = tc::sdesc_sw128(tc::smem_u32(sm + OFF_Q + buf * QBUF), 1024, 2048);
                    const uint64_t tO = tc::sdesc_sw128(tc::smem_u32(sm + OFF_DO + buf * QBUF), 1024, 2048);
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        const uint32_t acc = (ti > 0 || ks > 0) ? 1u : 0u;
                        tc::mma_bf16(tmem + COL_DV, tO + (uint64_t)((ks * 4096) >> 4),
                                     bWP + (uint64_t)((ks * 2048) >> 4), IDESC_T, acc);
                        tc::mma_bf16(tmem + COL_DK, tQ + (uint64_t)((ks * 4096) >> 4),
                                     bDS + (uint64_t)((ks * 2048) >> 4), IDESC_T, acc);
                    }
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc::mma_bf16(tmem + COL_DQ, aDS + (uint64_t)((kk * 32) >> 4),
                                     bKt + (uint64_t)((kk * 2048) >> 4), IDESC_DQ, kk > 0 ? 1u : 0u);
                    tc::mma_commit(o_bar);
                }
                // the next tile's S and U: behind this tile's products on the
                // tensor pipe, so they run during this tile's epilogue
                if (ti + 1 < sg.ntiles) {
                    if (!__all_sync(0xffffffffu, bt_wait(&tma_bar[nb], ptma[nb], s_abort))) { ok = false; break; }
                    ptma[nb] ^= 1u;
                    if (lane == 0) issue_su(ti + 1);
                }
                // this tile's products are done with its Q / dO buffer: the rows
                // of tile ti + 2 load into it
                if (!__all_sync(0xffffffffu, bt_wait(o_bar, po, s_abort))) { ok = false; break; }
                po ^= 1u;
                if (ti + 2 < sg.ntiles) load_rows(ti + 2);
            }
            if (sg.ntiles > 0) dkdv_held = true;
        }
    } else {
        // ------------------------------------------------------------ compute
        const int rt = tid & 127, hf = tid >> 7;          // tile row (TMEM lane), key half
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        float *red = (float *)(sm + OFF_RED);
        const int e = rt >> 3, h = rt & 7;
        uint32_t psu[2] = {0u, 0u}, po = 0u;
        for (int64_t sidx = blockIdx.x; sidx < nseg && ok; sidx += gridDim.x) {
            const BtSeg sg = bt_segment(p, sidx);
            const int64_t b = sg.b;
            const int g = sg.g;
            auto row_of = [&](int ti) -> BtRow {
                BtRow r;
                const int u = ti * BT_EPT + e;
                r.valid = u < sg.n_units;
                r.t = -1;
                r.slot = topk;
                if (r.valid) {
                    if (sg.own) {
                        r.t = sg.first + u;
                    } else {
                        const int32_t code = p.entries[sg.ebase + u];
                        r.t = code >> 5;
                        r.slot = code & 31;
                    }
                }
                return r;
            };
            // entry codes are read two tiles ahead and fusion weights one tile
            // ahead, so neither load's latency sits on a tile's critical path
            auto weight_of = [&](const BtRow &r) -> float {
                if (!r.valid) return 0.f;
                if (sg.own) return 1.f;
                return p.coef[((b * L + r.t) * H + (int64_t)g * G + h) * topk + r.slot].x;
            };
            BtRow cur = row_of(0);
            BtRow nxt = sg.ntiles > 1 ? row_of(1) : cur;
            float w_cur = weight_of(cur);
            for (int ti = 0; ti < sg.ntiles; ++ti) {
                const int buf = ti & 1;
                const bool more = ti + 1 < sg.ntiles;
                const BtRow nxt2 = ti + 2 < sg.ntiles ? row_of(ti + 2) : nxt;
                const float w_nxt = more ? weight_of(nxt) : 0.f;
                const bool valid = cur.valid;
                const int64_t t = cur.t;
                const int slot = cur.slot;
                const int64_t hrow = valid ? (b * L + t) * H + (int64_t)g * G + h : 0;
                const float w = w_cur;
                if (!cbar_and(bt_wait(&su_bar[buf], psu[buf], s_abort))) { ok = false; break; }
                psu[buf] ^= 1u;
                tc::fence_after_sync();
                // this row's chunk softmax, dw, dS and w p over this thread's 32
                // keys (j0 .. j0+31); the row max and the two sums are combined
                // with the other half through shared memory
                const int j0 = hf * 32;
                float s[32], uu[32];
                {
                    const uint32_t ts = tmem + lane_off + COL_SU + 128u * (uint32_t)buf + (uint32_t)j0;
                    tc::tmem_ld32(ts, s);
                    tc::tmem_ld32(ts + 64, uu);
                    tc::tmem_wait_ld();
                }
                const int nk = sg.own ? (valid ? (int)(t - sg.first) + 1 : 64) : 64;
                float mx = -INFINITY;
#pragma unroll
                for (int j = 0; j < 32; ++j) mx = j0 + j < nk ? fmaxf(mx, s[j]) : mx;
                red[hf * 128 + rt] = mx;
                cbar();
                mx = fmaxf(red[rt], red[128 + rt]);
                // exp(scale (s - max)) as 2^(scale log2(e) (s - max)) on the MUFU unit
                const float sl2 = p.scale * 1.4426950408889634f, ml2 = -sl2 * mx;
                float z = 0.f, zu = 0.f;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const float ej = j0 + j < nk ? tc::ex2_approx(fmaf(s[j], sl2, ml2)) : 0.f;
                    s[j] = ej;
                    z += ej;
                    zu = fmaf(ej, uu[j], zu);
                }
                red[256 + hf * 128 + rt] = z;
                red[512 + hf * 128 + rt] = zu;
                cbar();
                z = red[256 + rt] + red[384 + rt];
                zu = red[512 + rt] + red[640 + rt];
                const float inv = 1.f / z;
                const float dwv = zu * inv;
                if (valid && hf == 0) p.dw[hrow * (topk + 1) + slot] = dwv;
                const float fds = valid ? p.scale * w * inv : 0.f, fwp = valid ? w * inv : 0.f;
#pragma unroll
                for (int cq = 0; cq < 4; ++cq) {
                    uint32_t ds4[4], wp4[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int j = cq * 8 + 2 * i;
                        ds4[i] = pack2_bf16(fds * s[j] * (uu[j] - dwv), fds * s[j + 1] * (uu[j + 1] - dwv));
                        wp4[i] = pack2_bf16(fwp * s[j], fwp * s[j + 1]);
                    }
                    const uint32_t off = tc::sw128_offset(rt, hf * 4 + cq);
                    *reinterpret_cast<uint4 *>(sm + OFF_DS + off) = make_uint4(ds4[0], ds4[1], ds4[2], ds4[3]);
                    *reinterpret_cast<uint4 *>(sm + OFF_WP + off) = make_uint4(wp4[0], wp4[1], wp4[2], wp4[3]);
                }
                // dS and w P are complete for this warp; the S / U slot is read
                tc::fence_proxy_async_smem();
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(ds_full);
                if (!cbar_and(bt_wait(o_bar, po, s_abort))) { ok = false; break; }
                po ^= 1u;
                tc::fence_after_sync();
                // this row's dQ partial (fp16: 2^-11 relative, below the bf16
                // rounding of dS it already carries), each half 64 columns,
                // straight from registers: a lane's 32-byte pieces are whole
                // sectors, so no staging and no bulk copies
                const int64_t qrow = valid ? (((b * L + t) * p.Hkv + g) * (topk + 1) + slot) * G + h : 0;
                __half *dst = p.dqp + qrow * D;
#pragma unroll 1
                for (int cb = hf * 2; cb < hf * 2 + 2; ++cb) {
                    float v[32];
                    tc::tmem_ld32(tmem + lane_off + COL_DQ + cb * 32, v);
                    tc::tmem_wait_ld();
                    if (valid) {
#pragma unroll
                        for (int hq = 0; hq < 2; ++hq) {
                            uint32_t w8[8];
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                __half2 hv = __floats2half2_rn(v[16 * hq + 2 * i], v[16 * hq + 2 * i + 1]);
                                w8[i] = *reinterpret_cast<uint32_t *>(&hv);
                            }
                            asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
                                         :: "l"(dst + cb * 32 + hq * 16), "r"(w8[0]), "r"(w8[1]), "r"(w8[2]),
                                            "r"(w8[3]), "r"(w8[4]), "r"(w8[5]), "r"(w8[6]), "r"(w8[7])
                                         : "memory");
                        }
                    }
                }
                cur = nxt;
                nxt = nxt2;
                w_cur = w_nxt;
            }
            if (!ok) break;
            // the segment's dK and dV partials (thread = element of d; each half
            // 32 keys); dl is written by bwd_dl_kernel
            {
                float *pk = p.part + sidx * (int64_t)(129 * D);
                const int cb = hf;
                const bool any = sg.ntiles > 0;
                float vk[32], vv[32];
                if (any) {
                    tc::tmem_ld32(tmem + lane_off + COL_DK + cb * 32, vk);
                    tc::tmem_ld32(tmem + lane_off + COL_DV + cb * 32, vv);
                    tc::tmem_wait_ld();
                }
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    pk[(cb * 32 + j) * D + rt] = any ? vk[j] : 0.f;
                    pk[64 * D + (cb * 32 + j) * D + rt] = any ? vv[j] : 0.f;
                }
                if (any) {                   // TMEM dK / dV free for the next segment
                    tc::fence_before_sync();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(seg_free);
                }
            }
        }
    }
    if (!ok) *s_abort = 1;
    __syncthreads();
    if (*s_abort) {
        if (tid == 0) atomicOr(p.status, kFlagTimeout);
        // let copies and MMAs that may still be in flight land before exiting
        const long long t0 = clock64();
        while (clock64() - t0 < 20000000) { }
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 0) tc::tmem_dealloc(tmem, BT_TMEM_COLS);
}

// ---------------------------------------------------------------- CUDA-core companions
// The companions work per (b, t, g), one warp each: the G = 8 heads of a token
// share its slots, so the landmark rows and slot indices are read once for all
// eight, and the (t, g) blocks of Q, dw, coef and the dQ partials are
// contiguous, so every load is a coalesced 8- or 16-byte one.

// Four or eight consecutive landmark elements as fp32 (one load, or two for
// eight fp32 values).
template <typename TL> __device__ __forceinline__ void lm_load4(const TL *p, float (&v)[4]);
template <> __device__ __forceinline__ void lm_load4<float>(const float *p, float (&v)[4]) {
    const float4 u = *reinterpret_cast<const float4 *>(p);
    v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
}
template <> __device__ __forceinline__ void lm_load4<__nv_bfloat16>(const __nv_bfloat16 *p, float (&v)[4]) {
    const uint2 u = *reinterpret_cast<const uint2 *>(p);
    v[0] = __uint_as_float(u.x << 16); v[1] = __uint_as_float(u.x & 0xffff0000u);
    v[2] = __uint_as_float(u.y << 16); v[3] = __uint_as_float(u.y & 0xffff0000u);
}
template <typename TL> __device__ __forceinline__ void lm_load8(const TL *p, float (&v)[8]) {
    float a[4], b[4];
    lm_load4<TL>(p, a);
    lm_load4<TL>(p + 4, b);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[i] = a[i];
        v[4 + i] = b[i];
    }
}
template <> __device__ __forceinline__ void lm_load8<__nv_bfloat16>(const __nv_bfloat16 *p, float (&v)[8]) {
    Vec16<__nv_bfloat16>::unpack(*reinterpret_cast<const uint4 *>(p), v);
}

// Fusion weights w = softmax over the valid slots of scale q_h . l_k, written
// to coef[.].x.  Lane l holds elements 4l .. 4l+3 of the eight heads' queries
// and, for a group of four slots, of their four landmark rows: 32 partial dot
// products (slot-major), which five halving exchanges reduce over the warp so
// that lane l ends with the logit of slot 4i + l/8, head l%8.  A head's
// softmax then runs over the four lanes that share l%8 and over the groups.
template <typename TL>
__global__ void __launch_bounds__(256)
bwd_coefw_kernel(const __nv_bfloat16 *__restrict__ Q, const TL *__restrict__ lm,
                 const int32_t *__restrict__ idx, int64_t pairs, int H, int Hkv, int64_t L, int S,
                 int64_t Nc, int topk, float scale, float2 *__restrict__ coef,
                 unsigned *__restrict__ status) {
    constexpr int D = BT_D, G = BT_G, NGR = 8;    // topk <= 32: up to eight groups of four slots
    const int lane = threadIdx.x & 31;
    const int64_t tg = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);     // (b, t, g)
    if (tg >= pairs) return;
    const int g = (int)(tg % Hkv);
    const int64_t bt = tg / Hkv;
    const int64_t b = bt / L, t = bt % L;
    const int64_t bg = b * Hkv + g;
    const int64_t hrow0 = bt * H + (int64_t)g * G;
    float qv[G][4];
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
        const uint2 u = *reinterpret_cast<const uint2 *>(Q + (hrow0 + hh) * D + 4 * lane);
        qv[hh][0] = __uint_as_float(u.x << 16); qv[hh][1] = __uint_as_float(u.x & 0xffff0000u);
        qv[hh][2] = __uint_as_float(u.y << 16); qv[hh][3] = __uint_as_float(u.y & 0xffff0000u);
    }
    const int32_t ci_l = lane < topk ? idx[tg * topk + lane] : -1;
    const bool vk = ci_l >= 0 && (int64_t)ci_l < Nc && (int64_t)ci_l < t / S;
    if (lane < topk && ci_l >= 0 && !vk) atomicOr(status, kFlagBadIdx);
    const unsigned vmask = __ballot_sync(0xffffffffu, vk);
    float z[NGR];
#pragma unroll
    for (int gi = 0; gi < NGR; ++gi) {
        z[gi] = -INFINITY;
        if (gi * 4 >= topk) continue;                          // warp-uniform
        float v[32];
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            const int k = gi * 4 + kk;
            const int32_t ci = __shfl_sync(0xffffffffu, ci_l, k);
            float lv[4] = {0.f, 0.f, 0.f, 0.f};
            if ((vmask >> k) & 1u) lm_load4<TL>(lm + (bg * Nc + ci) * D + 4 * lane, lv);
#pragma unroll
            for (int hh = 0; hh < G; ++hh)
                v[kk * G + hh] = fmaf(qv[hh][3], lv[3], fmaf(qv[hh][2], lv[2], fmaf(qv[hh][1], lv[1], qv[hh][0] * lv[0])));
        }
        // after the exchange with offset o a lane keeps the half of its values
        // whose index bit matches its lane bit o, adding the partner's copy
#pragma unroll
        for (int st = 0; st < 5; ++st) {
            const int o = 16 >> st;
            const bool up = (lane & o) != 0;
#pragma unroll
            for (int i = 0; i < o; ++i) {
                const float send = up ? v[i] : v[i + o];
                const float keep = up ? v[i + o] : v[i];
                v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
            }
        }
        if ((vmask >> (gi * 4 + (lane >> 3))) & 1u) z[gi] = scale * v[0];
    }
    float m = -INFINITY;
#pragma unroll
    for (int gi = 0; gi < NGR; ++gi) m = fmaxf(m, z[gi]);
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
    float ew[NGR], sw = 0.f;
#pragma unroll
    for (int gi = 0; gi < NGR; ++gi) {
        ew[gi] = z[gi] > -INFINITY ? expf(z[gi] - m) : 0.f;
        sw += ew[gi];
    }
    sw += __shfl_xor_sync(0xffffffffu, sw, 8);
    sw += __shfl_xor_sync(0xffffffffu, sw, 16);
    float2 *cr = coef + (hrow0 + (lane & 7)) * topk;
#pragma unroll
    for (int gi = 0; gi < NGR; ++gi) {
        const int k = gi * 4 + (lane >> 3);
        if (k < topk) cr[k] = make_float2(z[gi] > -INFINITY ? ew[gi] / sw : 0.f, 0.f);
    }
}

// Per (b, t, g): dz = w (dw - sum w dw) per head and slot (to coef[.].y), and
// each head's dQ = the sum of its dQ partials over the valid slots and the own
// chunk + scale sum_k dz_k l_k.  The partials of (t, g) are one [slot][G][D]
// fp16 block: lane l reads the 16-byte pieces l + 32 j (j < 4) of a slot, i.e.
// elements 8 (l % 16) .. +8 of head 2j + l / 16.
template <typename TL>
__global__ void __launch_bounds__(256)
bwd_rowfin_kernel(const TL *__restrict__ lm, const int32_t *__restrict__ idx,
                  const float *__restrict__ dw, const __half *__restrict__ dqp, int64_t pairs,
                  int H, int Hkv, int64_t L, int S, int64_t Nc, int topk, int own_chunk,
                  float scale, float2 *__restrict__ coef, float *__restrict__ dQ) {
    constexpr int D = BT_D, G = BT_G;
    const int lane = threadIdx.x & 31;
    const int64_t tg = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);     // (b, t, g)
    if (tg >= pairs) return;
    const int g = (int)(tg % Hkv);
    const int64_t bt = tg / Hkv;
    const int64_t b = bt / L, t = bt % L;
    const int64_t bg = b * Hkv + g;
    const int64_t hrow0 = bt * H + (int64_t)g * G;
    const int32_t ci_l = lane < topk ? idx[tg * topk + lane] : -1;
    const bool vk = lane < topk && ci_l >= 0 && (int64_t)ci_l < Nc && (int64_t)ci_l < t / S;
    const unsigned vmask = __ballot_sync(0xffffffffu, vk);
    // lane k: dz of slot k for every head
    float wk[G], dwk[G], dzr[G];
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
        wk[hh] = vk ? coef[(hrow0 + hh) * topk + lane].x : 0.f;
        dwk[hh] = vk ? dw[(hrow0 + hh) * (topk + 1) + lane] : 0.f;
    }
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
        float dsum = wk[hh] * dwk[hh];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, o);
        dzr[hh] = wk[hh] * (dwk[hh] - dsum);
        if (lane < topk) coef[(hrow0 + hh) * topk + lane] = make_float2(wk[hh], dzr[hh]);
    }
    const int hs = lane >> 4, d0 = 8 * (lane & 15);
    float acc[4][8];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[j][e] = 0.f;
    const uint4 *qp = reinterpret_cast<const uint4 *>(dqp + tg * (int64_t)(topk + 1) * (G * D)) + lane;
    // the own chunk's partials and the next valid slot's loads go out before
    // the current slot is added (the slots are still added in index order)
    uint4 ro[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
        ro[j] = own_chunk ? qp[(int64_t)topk * (G * D / 8) + 32 * j] : make_uint4(0u, 0u, 0u, 0u);
    auto load_slot = [&](int k, uint4 (&r)[4], float (&l)[8]) {
        const int32_t ci = __shfl_sync(0xffffffffu, ci_l, k);
#pragma unroll
        for (int j = 0; j < 4; ++j) r[j] = qp[(int64_t)k * (G * D / 8) + 32 * j];
        lm_load8<TL>(lm + (bg * Nc + ci) * D + d0, l);
    };
    unsigned rest = vmask;                                   // warp-uniform
    int k = rest ? __ffs(rest) - 1 : -1;
    uint4 raw[4];
    float lv[8];
    if (k >= 0) {
        rest &= rest - 1;
        load_slot(k, raw, lv);
    }
    while (k >= 0) {
        const int kn = rest ? __ffs(rest) - 1 : -1;
        uint4 rawn[4];
        float lvn[8];
        if (kn >= 0) {
            rest &= rest - 1;
            load_slot(kn, rawn, lvn);
        }
        float dzk[G];
#pragma unroll
        for (int hh = 0; hh < G; ++hh) dzk[hh] = scale * __shfl_sync(0xffffffffu, dzr[hh], k);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float dz = hs ? dzk[2 * j + 1] : dzk[2 * j];
            const __half2 *h2 = reinterpret_cast<const __half2 *>(&raw[j]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __half22float2(h2[e]);
                acc[j][2 * e] += f.x + dz * lv[2 * e];
                acc[j][2 * e + 1] += f.y + dz * lv[2 * e + 1];
            }
        }
        k = kn;
        if (kn >= 0) {
#pragma unroll
            for (int j = 0; j < 4; ++j) raw[j] = rawn[j];
#pragma unroll
            for (int e = 0; e < 8; ++e) lv[e] = lvn[e];
        }
    }
    if (own_chunk) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const __half2 *h2 = reinterpret_cast<const __half2 *>(&ro[j]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __half22float2(h2[e]);
                acc[j][2 * e] += f.x;
                acc[j][2 * e + 1] += f.y;
            }
        }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float4 *dst = reinterpret_cast<float4 *>(dQ + (hrow0 + 2 * j + hs) * D + d0);
        dst[0] = make_float4(acc[j][0], acc[j][1], acc[j][2], acc[j][3]);
        dst[1] = make_float4(acc[j][4], acc[j][5], acc[j][6], acc[j][7]);
    }
}

// Landmark-gradient partial of each entry segment, dl = scale sum over its
// entries' head rows of dz q: one block per segment, warp w takes the entries
// w, w + 8, ... (lane l: elements 4l .. 4l+3 of the eight head rows, one
// 8-byte load each; lanes 0-7 load the entry's eight dz and broadcast them);
// the warps' sums are added in warp order.  Own-chunk segments carry none.
constexpr int kDlWarps = 8;
__global__ void __launch_bounds__(32 * kDlWarps)
bwd_dl_kernel(const __nv_bfloat16 *__restrict__ Q, const float2 *__restrict__ coef,
              const int32_t *__restrict__ entries, const int4 *__restrict__ segs,
              const int32_t *__restrict__ nseg_p, int H, int Hkv, int64_t L, int64_t NcAll,
              int topk, float scale, float *__restrict__ part) {
    constexpr int D = BT_D, G = BT_G;
    __shared__ float red[kDlWarps][D];
    const int64_t sidx = blockIdx.x;
    if (sidx >= *nseg_p) return;
    const int4 sg = segs[sidx];
    const int64_t bg = (int64_t)sg.x / NcAll;
    const int64_t b = bg / Hkv;
    const int g = (int)(bg % Hkv);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (!sg.w) {
#pragma unroll 2
        for (int u = warp; u < sg.z; u += kDlWarps) {
            const int32_t code = entries[sg.y + u];
            const int64_t r0 = (b * L + (code >> 5)) * H + (int64_t)g * G;
            const float dzl = lane < G ? coef[(r0 + lane) * topk + (code & 31)].y : 0.f;
            uint2 qr[G];
#pragma unroll
            for (int hh = 0; hh < G; ++hh)
                qr[hh] = *reinterpret_cast<const uint2 *>(Q + (r0 + hh) * D + 4 * lane);
#pragma unroll
            for (int hh = 0; hh < G; ++hh) {
                const float dz = __shfl_sync(0xffffffffu, dzl, hh);
                acc[0] = fmaf(dz, __uint_as_float(qr[hh].x << 16), acc[0]);
                acc[1] = fmaf(dz, __uint_as_float(qr[hh].x & 0xffff0000u), acc[1]);
                acc[2] = fmaf(dz, __uint_as_float(qr[hh].y << 16), acc[2]);
                acc[3] = fmaf(dz, __uint_as_float(qr[hh].y & 0xffff0000u), acc[3]);
            }
        }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) red[warp][4 * lane + e] = acc[e];
    __syncthreads();
    if (threadIdx.x < D) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < kDlWarps; ++w) s += red[w][threadIdx.x];
        part[sidx * (int64_t)(129 * D) + 128 * D + threadIdx.x] = scale * s;
    }
}

// ---------------------------------------------------------------- host side
bool backward_tc_supported(bool bf16, int G, int d) {
    return bf16 && G == BT_G && d == BT_D && encode_fn() != nullptr;
}

cudaError_t launch_backward_tc(const void *Q, const void *K, const void *V, const void *dO,
                               const void *lm, bool lm_bf16, const int32_t *idx, int B, int H,
                               int Hkv, int64_t L, int S, int64_t Nc, int64_t NcAll, int topk,
                               int own_chunk, float scale, float2 *coef, float *dw, __half *dqp,
                               const int4 *segs, const int32_t *nseg, const int32_t *entries,
                               float *part, int64_t max_seg, unsigned *status, float *dQ,
                               int phase, cudaStream_t st) {
    const int64_t rows = (int64_t)B * L * H;
    const int64_t pairs = (int64_t)B * L * Hkv;              // one warp per (b, t, g)
    const unsigned rblocks = (unsigned)((pairs + 7) / 8);
    cudaError_t e;
    if (phase == 0) {            // fusion weights (before the key pass)
        if (lm_bf16)
            bwd_coefw_kernel<__nv_bfloat16><<<rblocks, 256, 0, st>>>(
                (const __nv_bfloat16 *)Q, (const __nv_bfloat16 *)lm, idx, pairs, H, Hkv, L, S, Nc,
                topk, scale, coef, status);
        else
            bwd_coefw_kernel<float><<<rblocks, 256, 0, st>>>(
                (const __nv_bfloat16 *)Q, (const float *)lm, idx, pairs, H, Hkv, L, S, Nc, topk,
                scale, coef, status);
        return cudaGetLastError();
    }
    CUtensorMap mq, mo, mk, mv;
    if (!make_map_q3d(&mq, Q, (uint64_t)rows, BT_D, BT_G) ||
        !make_map_q3d(&mo, dO, (uint64_t)rows, BT_D, BT_G) ||
        !make_map(&mk, K, (uint64_t)B * Hkv * L, BT_D, 64) ||
        !make_map(&mv, V, (uint64_t)B * Hkv * L, BT_D, 64))
        return cudaErrorInvalidValue;
    BtParams p;
    p.segs = segs; p.nseg = nseg; p.entries = entries; p.coef = coef; p.dw = dw; p.dqp = dqp;
    p.part = part; p.status = status; p.L = L; p.NcAll = NcAll; p.H = H; p.Hkv = Hkv;
    p.topk = topk; p.S = S; p.scale = scale;
    e = cudaFuncSetAttribute(bwd_key_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             BT_SMEM);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t grid = max_seg < (int64_t)sms ? max_seg : (int64_t)sms;   // persistent
    bwd_key_tc_kernel<<<(unsigned)grid, kBtThreads, BT_SMEM, st>>>(mq, mo, mk, mv, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (lm_bf16)
        bwd_rowfin_kernel<__nv_bfloat16><<<rblocks, 256, 0, st>>>(
            (const __nv_bfloat16 *)lm, idx, dw, dqp, pairs, H, Hkv, L, S, Nc, topk, own_chunk, scale,
            coef, dQ);
    else
        bwd_rowfin_kernel<float><<<rblocks, 256, 0, st>>>(
            (const float *)lm, idx, dw, dqp, pairs, H, Hkv, L, S, Nc, topk, own_chunk, scale, coef,
            dQ);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    bwd_dl_kernel<<<(unsigned)max_seg, 32 * kDlWarps, 0, st>>>((const __nv_bfloat16 *)Q, coef, entries, segs,
                                                     nseg, H, Hkv, L, NcAll, topk, scale, part);
    return cudaGetLastError();
}

}  // namespace hsa
