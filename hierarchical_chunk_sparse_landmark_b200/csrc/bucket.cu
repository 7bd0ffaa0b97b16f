// bucket.cu -- chunk-bucketed work lists for the tensor-core prefill path.
//
// The selection gives every (b, t, g) up to K chunks.  To run the in-chunk
// attention as dense tensor-core tiles, entries (t, k) are grouped by the
// chunk they selected: a tile is one chunk's K/V and up to 128/G entries
// (G query-head rows each) that chose it, so each chunk's K/V is read once per
// tile instead of once per query.  Three passes over the selection:
//   count   -- entries per (b, g, chunk)               (shared-memory histogram)
//   scan    -- bucket offsets, tile descriptors        (one block per (b, g))
//   scatter -- entry ids into their bucket slots       (atomic cursors)
// The order of entries inside a bucket is not fixed, which does not change any
// result: every tile row is computed independently of the other rows.
#include "common.cuh"

namespace hsa {

constexpr int kBucketThreads = 256;
constexpr int kScanThreads = 1024;

// counts[bg * Nc + i] += #entries of (b, g) that selected chunk i
__global__ void __launch_bounds__(kBucketThreads)
bucket_count_kernel(const int32_t *__restrict__ idx, int Hkv, int64_t L, int topk, int64_t Nc,
                    int use_smem, int32_t *__restrict__ counts) {
    extern __shared__ int32_t hist[];
    const int g = blockIdx.y, b = blockIdx.z;
    const int64_t bg = (int64_t)b * Hkv + g;
    if (use_smem) {
        for (int64_t i = threadIdx.x; i < Nc; i += blockDim.x) hist[i] = 0;
        __syncthreads();
    }
    const int64_t t = (int64_t)blockIdx.x * kBucketThreads + threadIdx.x;
    if (t < L) {
        const int32_t *ip = idx + (((int64_t)b * L + t) * Hkv + g) * topk;
        for (int k = 0; k < topk; ++k) {
            const int32_t i = ip[k];
            if (i < 0) break;                       // padding only at the end
            if (use_smem) atomicAdd(&hist[i], 1);
            else atomicAdd(&counts[bg * Nc + i], 1);
        }
    }
    if (use_smem) {
        __syncthreads();
        for (int64_t i = threadIdx.x; i < Nc; i += blockDim.x)
            if (hist[i]) atomicAdd(&counts[bg * Nc + i], hist[i]);
    }
}

// One block per (b, g): exclusive scan of the counts -> absolute bucket
// offsets (cursor), tile descriptors appended at atomicAdd(tile_count).
// tiles[j] = {bg, chunk, first entry, n entries}
__global__ void __launch_bounds__(kScanThreads)
bucket_scan_kernel(const int32_t *__restrict__ counts, int Hkv, int64_t L, int topk, int64_t Nc,
                   int ept, int32_t *__restrict__ cursor, int4 *__restrict__ tiles,
                   int32_t *__restrict__ tile_count) {
    __shared__ int64_t warp_e[32], warp_t[32];
    __shared__ int64_t s_tile_base;
    const int g = blockIdx.x, b = blockIdx.y;
    const int64_t bg = (int64_t)b * Hkv + g;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t per = (Nc + kScanThreads - 1) / kScanThreads;
    const int64_t i0 = tid * per, i1 = (i0 + per < Nc) ? i0 + per : Nc;
    int64_t e_sum = 0, t_sum = 0;
    for (int64_t i = i0; i < i1; ++i) {
        const int64_t c = counts[bg * Nc + i];
        e_sum += c;
        t_sum += (c + ept - 1) / ept;
    }
    // block exclusive scan of (e_sum, t_sum)
    int64_t e_inc = e_sum, t_inc = t_sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int64_t a = __shfl_up_sync(0xffffffffu, e_inc, o);
        const int64_t c = __shfl_up_sync(0xffffffffu, t_inc, o);
        if (lane >= o) { e_inc += a; t_inc += c; }
    }
    if (lane == 31) { warp_e[warp] = e_inc; warp_t[warp] = t_inc; }
    __syncthreads();
    if (warp == 0) {
        int64_t a = warp_e[lane], c = warp_t[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int64_t x = __shfl_up_sync(0xffffffffu, a, o);
            const int64_t y = __shfl_up_sync(0xffffffffu, c, o);
            if (lane >= o) { a += x; c += y; }
        }
        warp_e[lane] = a;
        warp_t[lane] = c;
        if (lane == 31) s_tile_base = atomicAdd(tile_count, (int32_t)c);
    }
    __syncthreads();
    int64_t e_off = e_inc - e_sum + (warp ? warp_e[warp - 1] : 0);
    int64_t t_off = t_inc - t_sum + (warp ? warp_t[warp - 1] : 0) + s_tile_base;
    const int64_t base = bg * L * topk;
    for (int64_t i = i0; i < i1; ++i) {
        const int64_t c = counts[bg * Nc + i];
        cursor[bg * Nc + i] = (int32_t)(base + e_off);
        for (int64_t s = 0; s < c; s += ept) {
            const int64_t n = c - s < ept ? c - s : ept;
            tiles[t_off++] = make_int4((int)bg, (int)i, (int)(base + e_off + s), (int)n);
        }
        e_off += c;
    }
}

// entries[cursor[bg, i]++] = t * 32 + k
__global__ void __launch_bounds__(kBucketThreads)
bucket_scatter_kernel(const int32_t *__restrict__ idx, int Hkv, int64_t L, int topk, int64_t Nc,
                      int32_t *__restrict__ cursor, int32_t *__restrict__ entries) {
    const int g = blockIdx.y, b = blockIdx.z;
    const int64_t bg = (int64_t)b * Hkv + g;
    const int64_t t = (int64_t)blockIdx.x * kBucketThreads + threadIdx.x;
    if (t >= L) return;
    const int32_t *ip = idx + (((int64_t)b * L + t) * Hkv + g) * topk;
    for (int k = 0; k < topk; ++k) {
        const int32_t i = ip[k];
        if (i < 0) break;
        const int32_t p = atomicAdd(&cursor[bg * Nc + i], 1);
        entries[p] = (int32_t)(t * 32 + k);
    }
}

cudaError_t launch_bucket(const int32_t *idx, int B, int Hkv, int64_t L, int topk, int64_t Nc,
                          int ept, int32_t *counts, int32_t *cursor, int32_t *entries,
                          int4 *tiles, int32_t *tile_count, cudaStream_t st) {
    dim3 grid((unsigned)((L + kBucketThreads - 1) / kBucketThreads), (unsigned)Hkv, (unsigned)B);
    const int use_smem = Nc <= 8192 ? 1 : 0;
    const size_t smem = use_smem ? sizeof(int32_t) * (size_t)Nc : 0;
    bucket_count_kernel<<<grid, kBucketThreads, smem, st>>>(idx, Hkv, L, topk, Nc, use_smem,
                                                            counts);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    bucket_scan_kernel<<<dim3((unsigned)Hkv, (unsigned)B), kScanThreads, 0, st>>>(
        counts, Hkv, L, topk, Nc, ept, cursor, tiles, tile_count);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    bucket_scatter_kernel<<<grid, kBucketThreads, 0, st>>>(idx, Hkv, L, topk, Nc, cursor,
                                                           entries);
    return cudaGetLastError();
}

}  // namespace hsa
