// common.cuh -- device helpers shared by the libhsa kernels (not by the oracle).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

namespace hsa {

// ---------------------------------------------------------------- element access
template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Unpack one 16-byte vector of T into fp32 (8 bf16 or 4 fp32 elements).
template <typename T> struct Vec16;
template <> struct Vec16<float> {
    static constexpr int N = 4;
    __device__ __forceinline__ static void unpack(const uint4 &u, float *f) {
        f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
        f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
    }
};
template <> struct Vec16<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ __forceinline__ static void unpack(const uint4 &u, float *f) {
        // bf16 -> fp32 is exact: the bf16 bits are the top half of the fp32 bits.
        f[0] = __uint_as_float(u.x << 16); f[1] = __uint_as_float(u.x & 0xffff0000u);
        f[2] = __uint_as_float(u.y << 16); f[3] = __uint_as_float(u.y & 0xffff0000u);
        f[4] = __uint_as_float(u.z << 16); f[5] = __uint_as_float(u.z & 0xffff0000u);
        f[6] = __uint_as_float(u.w << 16); f[7] = __uint_as_float(u.w & 0xffff0000u);
    }
};

// ---------------------------------------------------------------- packed fp32 pairs
// Two fp32 values in one 64-bit register pair; ffma2 is an element-wise
// a * b + c with one rounding per element, exactly like two fmaf calls.
__device__ __forceinline__ uint64_t pack_f2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ float sum_f2(uint64_t v) {
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
    return lo + hi;
}
__device__ __forceinline__ void unpack_f2(uint64_t v, float &lo, float &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t add_f2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
// acc += q2 . (one 16-byte vector of T), q2 = the matching fp32 pairs.
template <typename T> struct Dot16;
template <> struct Dot16<float> {
    static constexpr int PAIRS = 2;
    __device__ __forceinline__ static uint64_t fma(const uint4 &u, const uint64_t *q2, uint64_t acc) {
        acc = ffma2(q2[0], pack_f2(__uint_as_float(u.x), __uint_as_float(u.y)), acc);
        return ffma2(q2[1], pack_f2(__uint_as_float(u.z), __uint_as_float(u.w)), acc);
    }
};
template <> struct Dot16<__nv_bfloat16> {
    static constexpr int PAIRS = 4;
    __device__ __forceinline__ static uint64_t pair(uint32_t w) {
        return pack_f2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
    }
    __device__ __forceinline__ static uint64_t fma(const uint4 &u, const uint64_t *q2, uint64_t acc) {
        acc = ffma2(q2[0], pair(u.x), acc);
        acc = ffma2(q2[1], pair(u.y), acc);
        acc = ffma2(q2[2], pair(u.z), acc);
        return ffma2(q2[3], pair(u.w), acc);
    }
};

// Streaming 16-byte load that does not allocate in L1 (read-once data).
__device__ __forceinline__ uint4 ld_stream16(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

// ---------------------------------------------------------------- selection keys
// A chunk candidate is one 64-bit key: the high word orders scores (larger is
// better), the low word holds ~index so that among equal scores the lower chunk
// index has the larger key.  Top-K = the K largest keys, whatever the order in
// which candidates were visited.  Key 0 is below every real candidate.
__device__ __forceinline__ uint32_t score_order_bits(float s) {
    uint32_t u = __float_as_uint(s);
    if (u == 0x80000000u) u = 0u;                 // -0 and +0 compare equal
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ uint64_t make_key(float s, int64_t idx) {
    return ((uint64_t)score_order_bits(s) << 32) | (uint64_t)(~(uint32_t)idx);
}
// Score of a key (inverse of score_order_bits); -inf for the empty key.
__device__ __forceinline__ float key_score(uint64_t k) {
    if (k == 0ull) return -INFINITY;
    const uint32_t h = (uint32_t)(k >> 32);
    return __uint_as_float((h & 0x80000000u) ? (h & 0x7fffffffu) : ~h);
}
__device__ __forceinline__ int32_t key_index(uint64_t k) {
    return k == 0ull ? -1 : (int32_t)(~(uint32_t)(k & 0xffffffffull));
}

// Warp-distributed sorted top-K list: lane k < topk holds the k-th best key.
// insert() is executed by the whole warp with the same x.
struct WarpTopK {
    uint64_t v;      // this lane's entry (0 = empty)
    int topk;
    __device__ __forceinline__ void init(int k) { v = 0ull; topk = k; }
    __device__ __forceinline__ uint64_t threshold() const {
        return __shfl_sync(0xffffffffu, v, topk - 1);
    }
    __device__ __forceinline__ void insert(uint64_t x) {
        const int lane = threadIdx.x & 31;
        const unsigned better = __ballot_sync(0xffffffffu, lane < topk && v > x);
        const int pos = __popc(better);
        const uint64_t up = __shfl_up_sync(0xffffffffu, v, 1);
        if (lane < topk) {
            if (lane == pos) v = x;
            else if (lane > pos) v = up;
        }
    }
};

// Sorted-list merging.  A warp register holds 32/KP lists (KP a power of two):
// lanes s*KP .. s*KP + KP - 1 hold list s in descending order (0 = empty).
// merge_lists returns, in the same layout, the KP best keys of the union of
// list s of `a` and list s of `b`: the element-wise maximum of a and b reversed
// is a bitonic sequence holding exactly those keys, and log2(KP) half-cleaner
// steps sort it.
__device__ __forceinline__ uint64_t merge_lists(uint64_t a, uint64_t b, int KP) {
    const int lane = threadIdx.x & 31;
    const int i = lane & (KP - 1);
    const uint64_t br = __shfl_sync(0xffffffffu, b, lane - i + (KP - 1 - i));
    uint64_t v = a > br ? a : br;
    for (int j = KP >> 1; j > 0; j >>= 1) {
        const uint64_t p = __shfl_xor_sync(0xffffffffu, v, j);
        v = (i & j) ? (v < p ? v : p) : (v > p ? v : p);
    }
    return v;
}
// Sort every KP-lane segment of a register in descending order (bitonic
// network; blocks of size k < KP alternate direction so that each pair forms
// a bitonic sequence, the last stage sorts every segment descending).
__device__ __forceinline__ uint64_t sort_segments_desc(uint64_t v, int KP) {
    const int lane = threadIdx.x & 31;
    for (int k = 2; k <= KP; k <<= 1)
        for (int j = k >> 1; j > 0; j >>= 1) {
            const uint64_t p = __shfl_xor_sync(0xffffffffu, v, j);
            const bool lower = (lane & j) == 0;
            const bool desc = k == KP || (lane & k) == 0;
            const uint64_t hi = v > p ? v : p, lo = v > p ? p : v;
            v = (lower == desc) ? hi : lo;
        }
    return v;
}
// Merge the 32/KP lists of one register into one (returned in every segment).
__device__ __forceinline__ uint64_t merge_segments(uint64_t v, int KP) {
    for (int m = KP; m < 32; m <<= 1) v = merge_lists(v, __shfl_xor_sync(0xffffffffu, v, m), KP);
    return v;
}
// Merge the lists of registers x[0 .. nr-1] (nr <= 8, warp-uniform) as a
// tree: the merges of one level are independent, so their shuffles overlap.
__device__ __forceinline__ uint64_t merge_regs8(uint64_t (&x)[8], int nr, int KP) {
#pragma unroll
    for (int w = 1; w < 8; w <<= 1)
#pragma unroll
        for (int i = 0; i + w < 8; i += 2 * w)
            if (i + w < nr) x[i] = merge_lists(x[i], x[i + w], KP);
    return x[0];
}
__host__ __device__ constexpr int pow2_at_least(int k) {
    return k <= 1 ? 1 : k <= 2 ? 2 : k <= 4 ? 4 : k <= 8 ? 8 : k <= 16 ? 16 : 32;
}

// ---------------------------------------------------------------- launch chaining
// Kernels of one call run in stream order.  A kernel launched with
// launch_pdl may be scheduled while its predecessor drains (programmatic
// dependent launch); it must call grid_dep_wait() before touching anything
// the predecessor writes (the wait returns once that grid has completed and
// its writes are visible; without a programmatic predecessor it returns at once).
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------- chunk geometry
// Chunks of S tokens, or variable-length chunks given by their boundaries
// (chunk c holds tokens bounds[c] .. bounds[c+1] - 1, at most 64 of them;
// tok_chunk[t] = the chunk holding token t).  The helpers clamp what they
// return to [0, L] and lengths to [0, 64], so that kernels stay inside their
// buffers whatever the boundaries hold (wrong boundaries are reported through
// the status word by varlen_setup_kernel).
struct Chunks {
    const int32_t *bounds;      // [n+1] or null: chunks of S tokens
    const int32_t *tok_chunk;   // [L]   or null
    int64_t L;
    int S;
};
constexpr int kMaxVarChunk = 64;
__device__ __forceinline__ int64_t chunk_first(const Chunks &c, int64_t i) {
    if (!c.bounds) return i * c.S;
    const int64_t f = c.bounds[i];
    return f < 0 ? 0 : f > c.L ? c.L : f;
}
__device__ __forceinline__ int chunk_len(const Chunks &c, int64_t i) {
    if (!c.bounds) return c.S;
    const int64_t n = (int64_t)c.bounds[i + 1] - c.bounds[i];
    return n < 0 ? 0 : n > kMaxVarChunk ? kMaxVarChunk : (int)n;
}
// Chunk holding token t: the chunks before it are the visible ones.
__device__ __forceinline__ int64_t chunk_of(const Chunks &c, int64_t t) {
    return c.tok_chunk ? (int64_t)c.tok_chunk[t] : t / c.S;
}

// ---------------------------------------------------------------- status word
// The first 256 bytes of every workspace.  word[0] = error flags set by kernels
// (bit 0: a bounded wait gave up).
constexpr size_t kStatusBytes = 256;
constexpr unsigned kFlagTimeout = 1u;
constexpr unsigned kFlagBadBounds = 2u;     // variable-length chunk boundaries invalid
constexpr unsigned kFlagBadIdx = 4u;        // backward: a selection entry names no visible chunk

__host__ __device__ constexpr size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Decode scratch inside the caller's workspace.  The ticket and unit-counter
// arrays sit right after the status word and must start at zero (the kernels
// leave them at zero); everything else is rewritten by every call.
struct DecodeScratch {
    unsigned *status;     // status word
    unsigned *tickets;    // [B*Hkv] scan blocks done
    unsigned *next_unit;  // [B*Hkv] next landmark unit to hand out
    int32_t *sel;         // [B*Hkv*topk] selected chunks
    uint64_t *cand;       // [B*Hkv*splits*topk] per-block candidate keys
};
// A decode over one shard of a cache cut into contiguous chunk ranges
// (context parallel); all zero / null for a whole cache.
struct DecodeShard {
    int64_t c0;            // global index of the shard's first chunk
    float *cand_score;     // [B*Hkv*topk] or null: the shard's top-K scores (scan)
    int32_t *cand_idx;     // [B*Hkv*topk] or null: their global chunk indices (-1: none)
    float *m, *Z, *acc;    // [B*H], [B*H], [B*H*d] or null: fusion state instead of O (attend)
    // ragged batch: sequence b sees its first lens[b] / S chunks (null: all of them)
    const int32_t *lens = nullptr;
    int S = 0;
};

// Bytes at the head of a decode workspace that must be zero before a call
// (status word, tickets, unit counters).
__host__ __device__ constexpr size_t decode_zero_head(int64_t B, int64_t Hkv) {
    return align_up(kStatusBytes + 2 * sizeof(unsigned) * (size_t)(B * Hkv), 256);
}

// Prefill backward (backward.cu): workspace layout and arguments.
struct BwdLayout {
    bool tc;                 // the tensor-core key pass (backward_tc.cu)
    int64_t BG, Nc, NcAll, TB, NTB, E, max_seg;
    size_t lm_off, coef_off, cnt_off, cnt_bytes, entries_off, segs_off, nseg_off, cseg_off,
        part_off, dw_off, dqp_off, total;
};
BwdLayout bwd_layout(int B, int H, int Hkv, int64_t L, int d, int S, int topk, bool dhsa,
                     bool tc);
bool backward_tc_supported(bool bf16, int G, int d);
struct BwdArgs {
    const void *Q, *K, *V, *dO, *lm;
    int lm_bf16, bf16, dhsa;
    const int32_t *idx;
    int B, H, Hkv, d, S, topk, own_chunk;
    int64_t L;
    float scale;
    float *dQ, *dK, *dV, *dlm;
    void *ws;
};
cudaError_t launch_backward(const BwdArgs &a, const BwdLayout &p, cudaStream_t st);

}  // namespace hsa
