// attend_tc.cu -- in-chunk attention and fusion on the 5th-generation tensor
// cores (tcgen05, TMEM accumulators, TMA tile loads), bf16 in, fp32 accumulate.
//
// HiLS Attention abstract: every query attends independently inside each
// retrieved chunk; the chunk outputs are fused with weights from the retrieval
// scores.  The work is chunk-bucketed (bucket.cu): a tile is one chunk's 64
// keys/values plus up to 128/G selected entries, each entry contributing its G
// query-head rows (the heads of a KV group share the selection), so a tile is a
// dense 128-row problem:
//
//   S = Q_rows . K_chunk^T          M=128, N=64, K=d   (tcgen05, TMEM)
//   P = exp(S*scale - rowmax)        per row, in registers (bf16 into smem)
//   O = P . V_chunk                  M=128, N=d, K=64   (tcgen05, TMEM)
//   partial[entry] = w/rowsum * O    fp16, one slot per (t, g, k)
//
// Mode "own": tiles of 128/G consecutive tokens of one chunk against their own
// chunk with the causal mask (keys c*S .. t); the epilogue adds the token's
// K partial slots and writes O in bf16, so the fusion needs no extra pass.
//
// One tile at a time per block of 128 threads (thread r <-> tile row r <->
// TMEM lane r); thread 0 issues TMA and MMA.  Two blocks fit per SM at d=128
// (80 KB of shared memory and 256 TMEM columns each; four at d=64), so one block's softmax and
// epilogue overlap the other's loads and MMAs.  Every wait is bounded; a
// timed-out block sets the workspace status flag, frees its TMEM and exits.
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
    static constexpr int A_BYTES = M * D * 2;    // gathered query rows
    static constexpr int KV_BYTES = 64 * D * 2;  // one chunk of K (or V)
    static constexpr int P_BYTES = M * 64 * 2;   // probabilities, bf16
    static constexpr int SMEM = 1024 + A_BYTES + 2 * KV_BYTES + P_BYTES + 64;
    // S: 64 fp32 columns at 0; O: D columns after it (power-of-two allocation)
    static constexpr uint32_t TMEM_COLS = D == 128 ? 256 : 128;
    static constexpr uint32_t O_COL = D == 128 ? 128 : 64;
};

struct TcParams {
    const int4 *tiles;
    const int32_t *tile_count;
    const int32_t *entries;
    const float *w;
    const int32_t *idx;
    __half *part;
    __nv_bfloat16 *O;
    unsigned *status;
    int64_t L;
    int64_t n_own_tiles;
    int H, Hkv, topk, S, own_mode;
    int add_own;          // own mode: 1 adds the causal own-chunk term, 0 only fuses
    float scale_log2e;
};

constexpr long long kWaitBudget = 4000000000LL;   // SM cycles (~2 s)

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}
__device__ __forceinline__ uint32_t pack_f16x2(float a, float b) {
    __half2 v = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}

template <int D, int G>
__global__ void __launch_bounds__(128, 1)
attend_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const TcParams p) {
    using C = TcCfg<D, G>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *sA = smem;                      // [KB][128 rows][128 B]
    uint8_t *sK = sA + C::A_BYTES;           // [KB][64 rows][128 B]
    uint8_t *sV = sK + C::KV_BYTES;          // [KB][64 rows][128 B]
    uint8_t *sP = sV + C::KV_BYTES;          // [128 rows][128 B]
    uint64_t *bar = (uint64_t *)(sP + C::P_BYTES);   // [0] loads, [1] mma
    uint32_t *s_tmem = (uint32_t *)(bar + 2);

    const int tid = threadIdx.x, warp = tid >> 5;
    if (warp == 0) {
        tc::tmem_alloc(s_tmem, C::TMEM_COLS);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        tc::mbar_init(&bar[0], 1);
        tc::mbar_init(&bar[1], 1);
        tc::fence_barrier_init();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *s_tmem;
    const uint32_t tS = tmem, tO = tmem + C::O_COL;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;

    constexpr uint32_t IDESC_S = tc::idesc_bf16_f32(128, 64, false);
    constexpr uint32_t IDESC_O = tc::idesc_bf16_f32(128, D, true);
    const int64_t L = p.L;
    const int S = p.S, H = p.H, Hkv = p.Hkv, topk = p.topk;
    const int64_t n_tiles = p.own_mode ? p.n_own_tiles
                                       : (int64_t)(*(volatile const int32_t *)p.tile_count);
    const int64_t own_per_bg = (L + C::EPT - 1) / C::EPT;
    uint32_t ph_load = 0, ph_mma = 0;
    int abort = 0;

    for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
        int64_t bg, first = 0, t0 = 0;
        int chunk, n;
        if (!p.own_mode) {
            const int4 d = p.tiles[tile];
            bg = d.x; chunk = d.y; first = d.z; n = d.w;
        } else {
            bg = tile / own_per_bg;
            t0 = (tile % own_per_bg) * C::EPT;
            n = (int)((L - t0) < C::EPT ? (L - t0) : C::EPT);
            chunk = (int)(t0 / S);
        }
        const int64_t b = bg / Hkv;
        const int g = (int)(bg % Hkv);

        // this thread's row: entry e, head h
        const int e = tid / G, h = tid % G;
        const bool valid = e < n;
        int64_t t = 0;
        int k = 0;
        if (valid) {
            if (!p.own_mode) {
                const int32_t code = p.entries[first + e];
                t = code >> 5;
                k = code & 31;
            } else {
                t = t0 + e;
            }
        }

        if (tid == 0) {
            tc::mbar_expect_tx(&bar[0], (uint32_t)(2 * C::KV_BYTES + n * G * D * 2));
            const int krow = (int)(bg * L + (int64_t)chunk * S);
#pragma unroll
            for (int kb = 0; kb < C::KB; ++kb) {
                tc::tma_load_2d(sK + kb * 8192, &tmK, &bar[0], kb * 64, krow);
                tc::tma_load_2d(sV + kb * 8192, &tmV, &bar[0], kb * 64, krow);
            }
            for (int ee = 0; ee < n; ++ee) {
                const int64_t tq = p.own_mode ? t0 + ee : (int64_t)(p.entries[first + ee] >> 5);
                const int qrow = (int)((b * L + tq) * H + (int64_t)g * G);
#pragma unroll
                for (int kb = 0; kb < C::KB; ++kb)
                    tc::tma_load_2d(sA + kb * (128 * 128) + ee * G * 128, &tmQ, &bar[0], kb * 64,
                                    qrow);
            }
        }
        if (!tc::mbar_wait(&bar[0], ph_load, kWaitBudget)) abort = 1;
        ph_load ^= 1;
        if (__syncthreads_or(abort)) break;

        // S = Q K^T
        if (tid == 0) {
            tc::fence_after_sync();
#pragma unroll
            for (int kb = 0; kb < C::KB; ++kb)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t ad = tc::sdesc_sw128(tc::smem_u32(sA + kb * 16384 + kk * 32), 16, 1024);
                    const uint64_t bd = tc::sdesc_sw128(tc::smem_u32(sK + kb * 8192 + kk * 32), 16, 1024);
                    tc::mma_bf16(tS, ad, bd, IDESC_S, (kb | kk) ? 1u : 0u);
                }
            tc::mma_commit(&bar[1]);
        }
        if (!tc::mbar_wait(&bar[1], ph_mma, kWaitBudget)) abort = 1;
        ph_mma ^= 1;
        tc::fence_after_sync();

        float s0[32], s1[32];
        tc::tmem_ld32(tS + lane_off + 0, s0);
        tc::tmem_ld32(tS + lane_off + 32, s1);
        tc::tmem_wait_ld();
        // causal limit inside the own chunk; all 64 keys of a retrieved chunk
        const int nk = (p.own_mode && valid) ? (int)(t - (int64_t)chunk * S) + 1 : 64;
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            if (j < nk) mx = fmaxf(mx, s0[j]);
            if (j + 32 < nk) mx = fmaxf(mx, s1[j]);
        }
        const float ms = mx * p.scale_log2e;
        float l = 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            s0[j] = j < nk ? tc::ex2_approx(fmaf(s0[j], p.scale_log2e, -ms)) : 0.f;
            s1[j] = j + 32 < nk ? tc::ex2_approx(fmaf(s1[j], p.scale_log2e, -ms)) : 0.f;
            l += s0[j] + s1[j];
        }
        // P row (unnormalised, bf16) into the swizzled K-major tile
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const float *src = c < 4 ? s0 + 8 * c : s1 + 8 * (c - 4);
            const uint4 u = make_uint4(pack_bf16x2(src[0], src[1]), pack_bf16x2(src[2], src[3]),
                                       pack_bf16x2(src[4], src[5]), pack_bf16x2(src[6], src[7]));
            *reinterpret_cast<uint4 *>(sP + tc::sw128_offset(tid, c)) = u;
        }
        float f = 0.f;
        if (valid) {
            const float wt = p.own_mode ? (float)p.add_own : p.w[((b * L + t) * H + (int64_t)g * G + h) * topk + k];
            f = wt / l;
        }
        tc::fence_proxy_async_smem();
        tc::fence_before_sync();
        __syncthreads();

        // O = P V
        if (tid == 0) {
            tc::fence_after_sync();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t ad = tc::sdesc_sw128(tc::smem_u32(sP + kk * 32), 16, 1024);
                const uint64_t bd = tc::sdesc_sw128(tc::smem_u32(sV + kk * 2048), 8192, 1024);
                tc::mma_bf16(tO, ad, bd, IDESC_O, kk ? 1u : 0u);
            }
            tc::mma_commit(&bar[1]);
        }
        if (!tc::mbar_wait(&bar[1], ph_mma, kWaitBudget)) abort = 1;
        ph_mma ^= 1;
        tc::fence_after_sync();

#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
            float o[32];
            tc::tmem_ld32(tO + lane_off + c0, o);
            tc::tmem_wait_ld();
            if (!valid) continue;
            if (!p.own_mode) {
                __half *dst = p.part + ((((b * L + t) * Hkv + g) * topk + k) * G + h) * (int64_t)D + c0;
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    reinterpret_cast<uint4 *>(dst)[q] = make_uint4(
                        pack_f16x2(o[8 * q + 0] * f, o[8 * q + 1] * f),
                        pack_f16x2(o[8 * q + 2] * f, o[8 * q + 3] * f),
                        pack_f16x2(o[8 * q + 4] * f, o[8 * q + 5] * f),
                        pack_f16x2(o[8 * q + 6] * f, o[8 * q + 7] * f));
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) o[j] *= f;
                const int32_t *ip = p.idx + ((b * L + t) * Hkv + g) * topk;
                for (int kk = 0; kk < topk; ++kk) {
                    if (ip[kk] < 0) break;
                    const __half *src = p.part + ((((b * L + t) * Hkv + g) * topk + kk) * G + h) * (int64_t)D + c0;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint4 u = reinterpret_cast<const uint4 *>(src)[q];
                        const __half2 *hh = reinterpret_cast<const __half2 *>(&u);
#pragma unroll
                        for (int z = 0; z < 4; ++z) {
                            const float2 v = __half22float2(hh[z]);
                            o[8 * q + 2 * z] += v.x;
                            o[8 * q + 2 * z + 1] += v.y;
                        }
                    }
                }
                __nv_bfloat16 *dst = p.O + ((b * L + t) * H + (int64_t)g * G + h) * D + c0;
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    reinterpret_cast<uint4 *>(dst)[q] = make_uint4(
                        pack_bf16x2(o[8 * q + 0], o[8 * q + 1]), pack_bf16x2(o[8 * q + 2], o[8 * q + 3]),
                        pack_bf16x2(o[8 * q + 4], o[8 * q + 5]), pack_bf16x2(o[8 * q + 6], o[8 * q + 7]));
            }
        }
        tc::fence_before_sync();
        if (__syncthreads_or(abort)) break;
    }

    if (abort) {
        // let copies and MMAs still in flight land before the block exits
        if (tid == 0) {
            tc::mbar_wait(&bar[0], ph_load ^ 1u, kWaitBudget);   // the phase that timed out
            atomicOr(p.status, kFlagTimeout);
        }
    }
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 0) tc::tmem_dealloc(tmem, C::TMEM_COLS);
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

template <int D, int G>
static cudaError_t launch_attend_tc_t(const void *Q, const void *K, const void *V, int B, int H,
                                      int Hkv, int64_t L, int S, int topk, int own_chunk,
                                      float scale, const int32_t *idx, const float *w, const int32_t *entries,
                                      const int4 *tiles, const int32_t *tile_count, int64_t max_tiles,
                                      __half *part, void *O, unsigned *status, int num_sms,
                                      cudaStream_t st) {
    using C = TcCfg<D, G>;
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, Q, (uint64_t)B * L * H, D, G) ||
        !make_map(&mk, K, (uint64_t)B * Hkv * L, D, 64) ||
        !make_map(&mv, V, (uint64_t)B * Hkv * L, D, 64))
        return cudaErrorInvalidValue;
    auto kern = attend_tc_kernel<D, G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    TcParams p;
    p.tiles = tiles; p.tile_count = tile_count; p.entries = entries; p.w = w; p.idx = idx;
    p.part = part; p.O = (__nv_bfloat16 *)O; p.status = status; p.L = L;
    p.H = H; p.Hkv = Hkv; p.topk = topk; p.S = S; p.add_own = own_chunk;
    p.scale_log2e = scale * 1.4426950408889634f;
    p.n_own_tiles = (int64_t)B * Hkv * ((L + C::EPT - 1) / C::EPT);
    // retrieved-chunk tiles (tile count known on the device only)
    p.own_mode = 0;
    int64_t grid = 2LL * num_sms;
    if (grid > max_tiles) grid = max_tiles > 0 ? max_tiles : 1;
    kern<<<(unsigned)grid, 128, C::SMEM, st>>>(mq, mk, mv, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // own-chunk tiles + fusion of the partials
    p.own_mode = 1;
    grid = 2LL * num_sms;
    if (grid > p.n_own_tiles) grid = p.n_own_tiles;
    kern<<<(unsigned)grid, 128, C::SMEM, st>>>(mq, mk, mv, p);
    return cudaGetLastError();
}

bool attend_tc_supported(bool bf16, int G, int d) {
    return bf16 && (G == 8 || G == 16) && (d == 64 || d == 128) && encode_fn() != nullptr;
}

cudaError_t launch_attend_tc(const void *Q, const void *K, const void *V, int B, int H, int Hkv,
                             int64_t L, int d, int S, int topk, int own_chunk, float scale,
                             const int32_t *idx, const float *w, const int32_t *entries,
                             const int4 *tiles, const int32_t *tile_count, int64_t max_tiles,
                             __half *part, void *O, unsigned *status, int num_sms,
                             cudaStream_t st) {
    const int G = H / Hkv;
#define HSA_TC(DD, GG) \
    return launch_attend_tc_t<DD, GG>(Q, K, V, B, H, Hkv, L, S, topk, own_chunk, scale, idx, w, entries, tiles, tile_count, max_tiles, part, O, status, num_sms, st)
    if (d == 128) { if (G == 8) HSA_TC(128, 8); HSA_TC(128, 16); }
    if (G == 8) HSA_TC(64, 8);
    HSA_TC(64, 16);
#undef HSA_TC
}

}  // namespace hsa
