// common.cuh -- device helpers shared by the libhsa kernels (not by the oracle).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

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

// ---------------------------------------------------------------- status word
// The first 256 bytes of every workspace.  word[0] = error flags set by kernels
// (bit 0: a bounded wait gave up).
constexpr size_t kStatusBytes = 256;
constexpr unsigned kFlagTimeout = 1u;

__host__ __device__ constexpr size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace hsa
