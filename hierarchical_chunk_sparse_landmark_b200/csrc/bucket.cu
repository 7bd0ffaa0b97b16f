// bucket.cu -- chunk-bucketed, token-windowed work lists for the tensor-core
// prefill path.
//
// The selection gives every (b, t, g) up to K chunks.  To run the in-chunk
// attention as dense tensor-core tiles, entries (t, k) are grouped by the
// chunk they selected: a tile is one chunk's K/V and up to 128/G entries (G
// query-head rows each) that chose it, so each chunk's K/V is read once per
// tile instead of once per query.  Grouping is done per token window (W
// consecutive tokens of one (b, g); one window spans the whole sequence unless
// the window count would exceed the work lists' limit).
//
// Passes over the selection (all windows at once):
//   count   -- entries per (window, chunk)                 (shared-memory histogram)
//   scan    -- bucket offsets, tile descriptors per window (one block per window)
//   fill    -- one launch, two kinds of blocks:
//              scatter: entry codes t*32+k into their bucket slots (atomic cursors)
//              flatten: one descriptor per queue position, each window's block
//                       taking its segment starts from the tile counts of the
//                       windows before it
// The order of entries inside a bucket is not fixed, which does not change
// any result: every tile row is computed independently of the other rows.
//
// Work queue (consumed by attend_tc.cu): segments C0, O0, C1, O1, ... where
// Cn = retrieved-chunk tiles of window n and On = own-chunk tiles of window n.
#include "common.cuh"

namespace hsa {

constexpr int kBucketThreads = 256;
constexpr int kScanThreads = 1024;

struct WinGeom {
    int64_t L, Nc, W, nwb;     // sequence length, chunks, window tokens, windows per (b, g)
    int Hkv, topk, ept;
    int64_t cap;               // tile capacity of one window's list
    Chunks ch;                 // chunks of S tokens or variable-length ones
};

__device__ __forceinline__ void window_span(const WinGeom &w, int64_t n, int64_t &bg,
                                            int64_t &t_start, int64_t &t_end) {
    bg = n / w.nwb;
    t_start = (n % w.nwb) * w.W;
    t_end = t_start + w.W < w.L ? t_start + w.W : w.L;
}

// counts[n * Nc + i] += #entries of window n that selected chunk i
__global__ void __launch_bounds__(kBucketThreads)
bucket_count_kernel(const int32_t *__restrict__ idx, WinGeom wg, int use_smem,
                    int32_t *__restrict__ counts) {
    grid_dep_wait();
    extern __shared__ int32_t hist[];
    const int g = blockIdx.y, b = blockIdx.z;
    const int64_t bg = (int64_t)b * wg.Hkv + g;
    const int64_t t_blk = (int64_t)blockIdx.x * kBucketThreads;    // within one window
    const int64_t n = bg * wg.nwb + t_blk / wg.W;
    if (use_smem) {
        for (int64_t i = threadIdx.x; i < wg.Nc; i += blockDim.x) hist[i] = 0;
        __syncthreads();
    }
    const int64_t t = t_blk + threadIdx.x;
    if (t < wg.L) {
        const int32_t *ip = idx + (((int64_t)b * wg.L + t) * wg.Hkv + g) * wg.topk;
        for (int k = 0; k < wg.topk; ++k) {
            const int32_t i = ip[k];
            if (i < 0) break;                       // padding only at the end
            if (use_smem) atomicAdd(&hist[i], 1);
            else atomicAdd(&counts[n * wg.Nc + i], 1);
        }
    }
    if (use_smem) {
        __syncthreads();
        for (int64_t i = threadIdx.x; i < wg.Nc; i += blockDim.x)
            if (hist[i]) atomicAdd(&counts[n * wg.Nc + i], hist[i]);
    }
}

// Own-chunk tiles of window n: the window's tokens cut at chunk starts (a
// tile's rows share its chunk's keys) into groups of at most ept tokens.
// With chunks of S tokens (a multiple of ept, windows start at multiples of
// 256) that is ceil(window tokens / ept).  Executed by one warp (lanes over
// the window's chunks); every lane returns the count.
__device__ __forceinline__ int64_t own_tile_count(const WinGeom &wg, int64_t n) {
    int64_t bg, ts, te;
    window_span(wg, n, bg, ts, te);
    if (!wg.ch.bounds) return (te - ts + wg.ept - 1) / wg.ept;
    const int lane = threadIdx.x & 31;
    const int64_t c_lo = chunk_of(wg.ch, ts), c_hi = chunk_of(wg.ch, te - 1);
    int64_t cnt = 0;
    for (int64_t c = c_lo + lane; c <= c_hi; c += 32) {
        const int64_t a = chunk_first(wg.ch, c), e = a + chunk_len(wg.ch, c);
        const int64_t lo = a > ts ? a : ts, hi = e < te ? e : te;
        if (hi > lo) cnt += (hi - lo + wg.ept - 1) / wg.ept;
    }
    for (int o = 16; o; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    return cnt;
}

// One block per window: cursor = absolute entry offset of each bucket, tile
// descriptors {bg, chunk, first entry, n entries} at wtiles[n * cap ...],
// wntiles[n] = number of tiles, wown[n] = own-chunk tiles, done[n] = 0.
__global__ void __launch_bounds__(kScanThreads)
bucket_scan_kernel(const int32_t *__restrict__ counts, WinGeom wg, int32_t *__restrict__ cursor,
                   int4 *__restrict__ wtiles, int32_t *__restrict__ wntiles,
                   int32_t *__restrict__ done, int32_t *__restrict__ wown) {
    grid_dep_wait();
    __shared__ int64_t warp_e[32], warp_t[32];
    const int64_t n = blockIdx.x;
    int64_t bg, t_start, t_end;
    window_span(wg, n, bg, t_start, t_end);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (warp == 1) {
        const int64_t no = own_tile_count(wg, n);
        if (lane == 0) wown[n] = (int32_t)no;
    }
    const int64_t Nc = wg.Nc;
    const int64_t per = (Nc + kScanThreads - 1) / kScanThreads;
    const int64_t i0 = tid * per, i1 = (i0 + per < Nc) ? i0 + per : Nc;
    const int32_t *cn = counts + n * Nc;
    int64_t e_sum = 0, t_sum = 0;
    for (int64_t i = i0; i < i1; ++i) {
        const int64_t c = cn[i];
        e_sum += c;
        t_sum += (c + wg.ept - 1) / wg.ept;
    }
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
        if (lane == 31) {
            wntiles[n] = (int32_t)c;
            done[n] = 0;
        }
    }
    __syncthreads();
    int64_t e_off = e_inc - e_sum + (warp ? warp_e[warp - 1] : 0);
    int64_t t_off = t_inc - t_sum + (warp ? warp_t[warp - 1] : 0);
    const int64_t base = bg * wg.L * wg.topk + t_start * wg.topk;     // window's entry region
    int4 *tl = wtiles + n * wg.cap;
    for (int64_t i = i0; i < i1; ++i) {
        const int64_t c = cn[i];
        cursor[n * Nc + i] = (int32_t)(base + e_off);
        for (int64_t s = 0; s < c; s += wg.ept) {
            const int64_t m = c - s < wg.ept ? c - s : wg.ept;
            tl[t_off++] = make_int4((int)bg, (int)i, (int)(base + e_off + s), (int)m);
        }
        e_off += c;
    }
}

// entries[cursor[n, i]++] = t * 32 + k.  A block's 256 tokens lie in one window
// (W is a multiple of 256).  With the chunk histogram in shared memory, each
// entry takes its rank within the block by a shared atomic, the block reserves
// each chunk's range with one global atomic, and the entries are written
// at base + rank.
__device__ __forceinline__ void bucket_scatter(const int32_t *__restrict__ idx, const WinGeom &wg,
                                               int use_smem, int64_t blk, int32_t *__restrict__ cursor,
                                               int32_t *__restrict__ entries, int32_t *hist) {
    // blk enumerates (token block, g, b) with the token block fastest
    const int64_t ntb = (wg.L + kBucketThreads - 1) / kBucketThreads;
    const int64_t tb = blk % ntb, bg = blk / ntb;
    const int g = (int)(bg % wg.Hkv), b = (int)(bg / wg.Hkv);
    const int64_t t = tb * kBucketThreads + threadIdx.x;
    const int64_t n = bg * wg.nwb + (tb * kBucketThreads) / wg.W;
    const int32_t *ip = idx + (((int64_t)b * wg.L + (t < wg.L ? t : 0)) * wg.Hkv + g) * wg.topk;
    if (!use_smem) {
        if (t >= wg.L) return;
        for (int k = 0; k < wg.topk; ++k) {
            const int32_t i = ip[k];
            if (i < 0) break;                       // padding only at the end
            const int32_t pos = atomicAdd(&cursor[n * wg.Nc + i], 1);
            entries[pos] = (int32_t)(t * 32 + k);
        }
        return;
    }
    for (int64_t i = threadIdx.x; i < wg.Nc; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    int32_t chunk[32], rank[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) {
        chunk[k] = -1;
        if (k < wg.topk && t < wg.L) chunk[k] = ip[k];
        rank[k] = chunk[k] >= 0 ? atomicAdd(&hist[chunk[k]], 1) : 0;
    }
    __syncthreads();
    for (int64_t i = threadIdx.x; i < wg.Nc; i += blockDim.x) {
        const int32_t c = hist[i];
        hist[i] = c ? atomicAdd(&cursor[n * wg.Nc + i], c) : 0;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 32; ++k)
        if (chunk[k] >= 0) entries[hist[chunk[k]] + rank[k]] = (int32_t)(t * 32 + k);
}

// Flat tile list: tiles[q] = descriptor of queue position q, so the consumer
// needs one load per tile instead of a search over segment starts.
// {bg, chunk, first entry, n} for retrieved-chunk tiles; own-chunk tiles are
// {bg, chunk, first token, n | kOwnTileFlag}.
// Window n's segments start after the tiles of windows 0 .. n-1 (queue order
// C0 O0 C1 O1 ...); the last window also writes the queue length.
constexpr int kOwnTileFlag = 1 << 30;
__device__ __forceinline__ void bucket_flatten(const int4 *__restrict__ wtiles,
                                               const int32_t *__restrict__ wntiles,
                                               const int32_t *__restrict__ wown, const WinGeom &wg,
                                               int64_t n, int64_t NW, int64_t *__restrict__ seg_start,
                                               int4 *__restrict__ tiles, int64_t *red) {
    int64_t part = 0;
    for (int64_t m = threadIdx.x; m < n; m += blockDim.x) part += wntiles[m] + wown[m];
    for (int o = 16; o; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = part;
    __syncthreads();
    int64_t c0 = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) c0 += red[w];
    const int nc = wntiles[n];
    const int64_t o0 = c0 + nc, no = wown[n];
    if (threadIdx.x == 0) {
        seg_start[2 * n] = c0;
        seg_start[2 * n + 1] = o0;
        if (n == NW - 1) seg_start[2 * NW] = o0 + no;
    }
    int64_t bg, ts, te;
    window_span(wg, n, bg, ts, te);
    for (int j = threadIdx.x; j < nc; j += blockDim.x) tiles[c0 + j] = wtiles[n * wg.cap + j];
    if (!wg.ch.bounds) {
        for (int64_t j = threadIdx.x; j < no; j += blockDim.x) {
            const int64_t t0 = ts + j * wg.ept;
            const int64_t cnt = te - t0 < wg.ept ? te - t0 : wg.ept;
            tiles[o0 + j] = make_int4((int)bg, (int)(t0 / wg.ch.S), (int)t0, (int)cnt | kOwnTileFlag);
        }
        return;
    }
    // variable-length chunks: warp 0 walks the window's chunks 32 at a time,
    // each lane emitting its chunk's tiles at its prefix offset
    if (threadIdx.x >= 32) return;
    const int lane = threadIdx.x;
    const int64_t c_lo = chunk_of(wg.ch, ts), c_hi = chunk_of(wg.ch, te - 1);
    int64_t base = o0;
    for (int64_t c0r = c_lo; c0r <= c_hi; c0r += 32) {
        const int64_t c = c0r + lane;
        int64_t lo = 0, hi = 0, k = 0;
        if (c <= c_hi) {
            const int64_t a = chunk_first(wg.ch, c), e = a + chunk_len(wg.ch, c);
            lo = a > ts ? a : ts;
            hi = e < te ? e : te;
            k = hi > lo ? (hi - lo + wg.ept - 1) / wg.ept : 0;
        }
        int64_t incl = k;
        for (int o = 1; o < 32; o <<= 1) {
            const int64_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        for (int64_t j = 0; j < k; ++j) {
            const int64_t t0 = lo + j * wg.ept;
            const int64_t cnt = hi - t0 < wg.ept ? hi - t0 : wg.ept;
            const int64_t q = base + incl - k + j;
            if (q < o0 + no) tiles[q] = make_int4((int)bg, (int)c, (int)t0, (int)cnt | kOwnTileFlag);
        }
        base += __shfl_sync(0xffffffffu, incl, 31);
    }
}

// Blocks [0, nscatter) scatter entries, blocks [nscatter, nscatter + NW) flatten
// one window each; both read only what bucket_scan_kernel wrote.
__global__ void __launch_bounds__(kBucketThreads)
bucket_fill_kernel(const int32_t *__restrict__ idx, WinGeom wg, int use_smem, int64_t nscatter,
                   int64_t NW, int32_t *__restrict__ cursor, int32_t *__restrict__ entries,
                   const int4 *__restrict__ wtiles, const int32_t *__restrict__ wntiles,
                   const int32_t *__restrict__ wown, int64_t *__restrict__ seg_start,
                   int4 *__restrict__ tiles) {
    grid_dep_wait();
    extern __shared__ int32_t hist[];             // [Nc] counts, then range bases
    __shared__ int64_t red[kBucketThreads / 32];
    const int64_t blk = blockIdx.x;
    if (blk < nscatter)
        bucket_scatter(idx, wg, use_smem, blk, cursor, entries, hist);
    else
        bucket_flatten(wtiles, wntiles, wown, wg, blk - nscatter, NW, seg_start, tiles, red);
}

cudaError_t launch_bucket(const int32_t *idx, int B, int Hkv, int64_t L, int topk, int64_t Nc,
                          int S, const int32_t *bounds, const int32_t *tok_chunk, int ept,
                          int64_t W, int64_t cap, int32_t *counts, int32_t *cursor,
                          int32_t *entries, int4 *wtiles, int32_t *wntiles, int32_t *done,
                          int32_t *wown, int64_t *seg_start, int4 *tiles, cudaStream_t st) {
    WinGeom wg;
    wg.L = L; wg.Nc = Nc; wg.W = W; wg.nwb = (L + W - 1) / W;
    wg.Hkv = Hkv; wg.topk = topk; wg.ept = ept; wg.cap = cap;
    wg.ch.bounds = bounds; wg.ch.tok_chunk = tok_chunk; wg.ch.L = L; wg.ch.S = S;
    const int64_t NW = (int64_t)B * Hkv * wg.nwb;
    dim3 grid((unsigned)((L + kBucketThreads - 1) / kBucketThreads), (unsigned)Hkv, (unsigned)B);
    const int use_smem = Nc <= 8192 ? 1 : 0;
    const size_t smem = use_smem ? sizeof(int32_t) * (size_t)(Nc > 0 ? Nc : 1) : 0;
    // the counts were zeroed before the selection: the count pass follows the
    // selection kernel as a programmatic dependent
    cudaError_t e = launch_pdl(bucket_count_kernel, grid, dim3(kBucketThreads), smem, st, idx, wg,
                               use_smem, counts);
    if (e != cudaSuccess) return e;
    e = launch_pdl(bucket_scan_kernel, dim3((unsigned)NW), dim3(kScanThreads), 0, st, counts, wg,
                   cursor, wtiles, wntiles, done, wown);
    if (e != cudaSuccess) return e;
    const int64_t nscatter = (int64_t)grid.x * grid.y * grid.z;
    if (NW == 0 && nscatter == 0) return cudaSuccess;
    return launch_pdl(bucket_fill_kernel, dim3((unsigned)(nscatter + NW)), dim3(kBucketThreads), smem, st,
                      idx, wg, use_smem, nscatter, NW, cursor, entries, (const int4 *)wtiles,
                      (const int32_t *)wntiles, (const int32_t *)wown, seg_start, tiles);
}

}  // namespace hsa
