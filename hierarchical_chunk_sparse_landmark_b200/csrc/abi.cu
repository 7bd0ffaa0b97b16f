// abi.cu -- the extern "C" entry points of libhsa (declared in include/hsa.h):
// argument validation, workspace layout and kernel dispatch.
#include <cuda_bf16.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "attend_tc.h"
#include "common.cuh"
#include "hsa.h"

namespace hsa {
cudaError_t launch_landmarks(const void *K, bool bf16, float *lm, int B, int Hkv, int64_t L,
                             int d, cudaStream_t st);
cudaError_t launch_select(const void *Q, bool q_bf16, const void *lm, bool lm_bf16, int B, int H,
                          int Hkv, int64_t L, int d, int S, int64_t Nc, const int32_t *bounds,
                          const int32_t *tok_chunk, int topk, float scale, int R, int pool_mean,
                          int32_t *idx, float *w, cudaStream_t st);
cudaError_t launch_attend_simt(const void *Q, const void *K, const void *V, bool bf16,
                               const int32_t *idx, const float *w, int B, int H, int Hkv,
                               int64_t L, int d, int S, int topk, int own_chunk, float scale,
                               int union_softmax, const int32_t *bounds, const int32_t *tok_chunk,
                               void *O, cudaStream_t st);
cudaError_t launch_varlen_setup(const int32_t *bounds, int64_t n, int64_t L, int32_t *bs,
                                int32_t *tok_chunk, unsigned *status, cudaStream_t st);
cudaError_t launch_landmarks_append(const void *K, bool bf16, void *lm, bool lm_bf16, int B,
                                    int Hkv, int64_t Lmax, int d, int S, const int32_t *len0,
                                    const int32_t *len1, int max_new_chunks, cudaStream_t st);
cudaError_t launch_landmarks_varlen(const void *K, bool bf16, float *lm, int B, int Hkv, int64_t L,
                                    int d, const int32_t *bounds, int64_t n, cudaStream_t st);
cudaError_t launch_decode(const void *q, const void *Kc, const void *Vc, bool bf16,
                          const void *lm, bool lm_bf16, int B, int H, int Hkv, int64_t Lc, int d,
                          int S, int topk, float scale, int splits, const DecodeScratch &ws,
                          void *O, int32_t *idx_out, const DecodeShard &sh, int stages,
                          const int32_t *sel, cudaStream_t st);
cudaError_t launch_decode_cp_merge(const float *score, const int32_t *cidx, int R, int B, int Hkv,
                                   int topk, int32_t *idx, cudaStream_t st);
cudaError_t launch_decode_cp_combine(const float *m, const float *Z, const float *acc, int R,
                                     int B, int H, int d, bool bf16, void *O, cudaStream_t st);
int decode_splits(int B, int Hkv, int64_t Nc, int num_sms);
bool select_tc_supported();
cudaError_t launch_split_landmarks(const void *lm, void *split, int64_t n, cudaStream_t st);
cudaError_t launch_select_tc(const void *Q, const void *lm, bool lm_bf16, const void *split, int B,
                             int H, int Hkv, int64_t L, int d, int S, int64_t Nc, int topk,
                             float scale, int R, int pool_mean, const int32_t *bounds,
                             const int32_t *tok_chunk, int32_t *idx, unsigned *status,
                             bool force_multi_tile, bool *multi, cudaStream_t st);
cudaError_t launch_bucket(const int32_t *idx, int B, int Hkv, int64_t L, int topk, int64_t Nc,
                          int S, const int32_t *bounds, const int32_t *tok_chunk, int ept,
                          int64_t W, int64_t cap, int32_t *counts, int32_t *cursor,
                          int32_t *entries, int4 *wtiles, int32_t *wntiles, int32_t *done,
                          int32_t *wown, int64_t *seg_start, int4 *tiles, cudaStream_t st);
cudaError_t launch_selftest_wait(unsigned *status, long long budget, cudaStream_t st);
// Status word of hsa_decode_noalloc's fixed array on the stream's device
// (decode_noalloc.cu); nullptr when the array is unused there and !mark.
hsa_status_t noalloc_status_word(cudaStream_t stream, bool mark, void **out);
}  // namespace hsa

using namespace hsa;

namespace {

constexpr int kChunk = 64;

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }
bool dtype_ok(hsa_dtype_t t) { return t == HSA_F32 || t == HSA_BF16; }

// Per-thread path overrides (hsa_set_path_overrides) and the kernels of the
// thread's last call (hsa_last_call_kernels).
thread_local int t_path_flags = 0;
thread_local int64_t t_window_tokens = 0;
thread_local unsigned t_kernels = 0;

// Shape checks shared by every call.  INVALID_ARG for impossible requests,
// UNSUPPORTED for valid ones this build does not implement.
hsa_status_t check_shape(int B, int H, int Hkv, int64_t L, int d, int S, int topk) {
    if (B < 1 || H < 1 || Hkv < 1 || L < 0 || d < 1 || S < 1 || topk < 1)
        return HSA_ERR_INVALID_ARG;
    if (H % Hkv != 0) return HSA_ERR_INVALID_ARG;
    const int G = H / Hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16) return HSA_ERR_UNSUPPORTED;
    if (d != 64 && d != 128) return HSA_ERR_UNSUPPORTED;
    if (S != kChunk) return HSA_ERR_UNSUPPORTED;
    if (topk > 32) return HSA_ERR_UNSUPPORTED;
    if (L > (int64_t)INT32_MAX) return HSA_ERR_UNSUPPORTED;   // chunk indices are int32
    return HSA_OK;
}

int num_sms() {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 148;
    return sms;
}

// Shapes the chunk-bucketed tensor-core path takes (bf16 inputs are checked
// at dispatch): G in {8, 16} so a 128-row tile holds whole KV groups, and all
// row / entry indices fit the 32-bit fields of the work lists and TMA maps.
bool tc_shape_ok(int B, int H, int Hkv, int64_t L, int d, int topk) {
    const int G = H / Hkv;
    if (!(G == 8 || G == 16) || !(d == 64 || d == 128)) return false;
    if (L >= (int64_t(1) << 26)) return false;                      // entry code t*32+k
    if ((int64_t)B * L * H >= INT32_MAX) return false;              // TMA row of Q
    if ((int64_t)B * Hkv * L * topk >= INT32_MAX) return false;     // entry index
    if ((int64_t)B * Hkv * Hkv >= (int64_t(1) << 32)) return false; // (b, g) split by a multiply
    return true;
}

// Token window of the work lists.  A window's tiles re-read each of its
// tokens' query rows once per selected chunk, spread over the window's whole
// run, so the window's query rows (W * G * d * 2 bytes) should stay in L2:
// windows of at most ~16 MB of them (8192 tokens at G = 8, d = 128), else one
// window per (b, g) -- bigger windows fill the chunk buckets better (on the
// L = 131072 prefill: 8192-token windows 3.01 ms, 16384 3.06, 32768 3.18,
// one window 3.55).  The
// window is a multiple of 256 tokens (the work-list blocks' size);
// hsa_set_path_overrides can set it (tests force several windows on small shapes).
int64_t tc_window(int B, int H, int Hkv, int64_t L, int d, int topk, int64_t max_windows) {
    (void)topk;
    int64_t W = (L + 255) / 256 * 256;
    const int64_t q_bytes_per_token = (int64_t)(H / Hkv) * d * 2;
    int64_t cap = (int64_t(16) << 20) / q_bytes_per_token / 256 * 256;
    if (t_window_tokens > 0) cap = t_window_tokens / 256 * 256;
    if (cap >= 256 && W > cap) W = cap;
    while ((int64_t)B * Hkv * ((L + W - 1) / W) > max_windows) W *= 2;
    return W;
}

struct PrefillLayout {
    size_t idx_off, w_off, lm_off, tokc_off, bnds_off, total;
    // tensor-core path (present when tc_shape_ok)
    bool tc;
    int64_t W, NW, cap;
    size_t counts_off, counts_bytes, cursor_off, entries_off, wtiles_off, wntiles_off, done_off,
        wown_off, seg_off, tiles_off, zf_off, ownf_off, ownm_off, part_off, own_off, lmsplit_off;
};

// Nc: chunks with a landmark (L / S, or the number of variable-length chunks).
PrefillLayout prefill_layout(int B, int H, int Hkv, int64_t L, int d, int S, int topk, int64_t Nc,
                             bool varlen) {
    PrefillLayout p;
    size_t off = kStatusBytes;
    p.idx_off = off;
    off = align_up(off + sizeof(int32_t) * (size_t)B * L * Hkv * topk, 256);
    p.w_off = off;
    off = align_up(off + sizeof(float) * (size_t)B * L * H * topk, 256);
    p.lm_off = off;
    off = align_up(off + sizeof(float) * (size_t)B * Hkv * Nc * d, 256);
    p.tokc_off = off;                // chunk of every token (variable-length chunks)
    if (varlen) off = align_up(off + sizeof(int32_t) * (size_t)L, 256);
    p.bnds_off = off;                // checked boundaries + outcome (variable-length chunks)
    if (varlen) off = align_up(off + sizeof(int32_t) * (size_t)(Nc + 2), 256);
    p.tc = tc_shape_ok(B, H, Hkv, L, d, topk);
    p.W = p.NW = p.cap = 0;
    p.counts_off = p.counts_bytes = p.cursor_off = p.entries_off = p.wtiles_off = 0;
    p.wntiles_off = p.done_off = p.wown_off = p.seg_off = p.tiles_off = p.part_off = p.own_off = 0;
    p.zf_off = p.ownf_off = p.ownm_off = p.lmsplit_off = 0;
    if (p.tc) {
        const int ept = 128 / (H / Hkv);
        p.W = tc_window(B, H, Hkv, L, d, topk, attend_tc_max_windows());
        p.NW = (int64_t)B * Hkv * ((L + p.W - 1) / p.W);
        p.cap = (p.W * topk + ept - 1) / ept + Nc;
        p.counts_off = off;
        p.counts_bytes = sizeof(int32_t) * (size_t)(p.NW * Nc > 0 ? p.NW * Nc : 1);
        off = align_up(off + p.counts_bytes, 256);
        p.cursor_off = off;
        off = align_up(off + p.counts_bytes, 256);
        p.entries_off = off;
        off = align_up(off + sizeof(int32_t) * (size_t)B * Hkv * L * topk, 256);
        p.wtiles_off = off;
        off = align_up(off + sizeof(int4) * (size_t)(p.NW * p.cap), 256);
        p.wntiles_off = off;
        off = align_up(off + sizeof(int32_t) * (size_t)p.NW, 256);
        p.done_off = off;
        off = align_up(off + sizeof(int32_t) * (size_t)p.NW, 256);
        p.wown_off = off;            // own-chunk tiles per window
        off = align_up(off + sizeof(int32_t) * (size_t)p.NW, 256);
        p.seg_off = off;
        off = align_up(off + sizeof(int64_t) * (size_t)(2 * p.NW + 1), 256);
        p.tiles_off = off;           // retrieved tiles + own-chunk tiles of every window
        // own-chunk tiles: a window's tokens in groups of ept, cut at chunk
        // starts as well with variable-length chunks (at most one per token)
        const int64_t own_cap = varlen ? p.W : (p.W + ept - 1) / ept;
        off = align_up(off + sizeof(int4) * (size_t)(p.NW * (p.cap + own_cap)), 256);
        p.zf_off = off;
        off = align_up(off + 2 * sizeof(float) * (size_t)B * L * H * topk, 256);
        p.ownf_off = off;
        off = align_up(off + sizeof(float) * (size_t)B * L * H, 256);
        p.ownm_off = off;            // own-chunk row maxima (union-softmax fusion)
        off = align_up(off + sizeof(float) * (size_t)B * L * H, 256);
        p.part_off = off;
        off = align_up(off + sizeof(__nv_bfloat16) * (size_t)B * L * H * topk * d, 256);
        p.own_off = off;
        off = align_up(off + sizeof(__nv_bfloat16) * (size_t)B * L * H * d, 256);
        p.lmsplit_off = off;         // fp32 landmarks as two bf16 planes (tensor-core path)
        off = align_up(off + 2 * sizeof(__nv_bfloat16) * (size_t)B * Hkv * Nc * d, 256);
    }
    p.total = off;
    return p;
}

bool force_simt_path() { return (t_path_flags & HSA_PATH_SIMT_PREFILL) != 0; }
// Selection on CUDA cores even where the tensor-core selection applies (A/B checks).
bool force_simt_select() { return (t_path_flags & HSA_PATH_SIMT_SELECT) != 0; }
bool force_multi_tile_select() { return (t_path_flags & HSA_PATH_MULTI_TILE_SELECT) != 0; }

// Decode workspace: status | tickets | unit counters (the zeroed head) | sel | cand.
struct DecodeLayout {
    size_t sel_off, cand_off, total;
    int64_t pairs;
    int splits;
    DecodeScratch at(char *ws) const {
        DecodeScratch s;
        s.status = (unsigned *)ws;
        s.tickets = (unsigned *)(ws + kStatusBytes);
        s.next_unit = s.tickets + pairs;
        s.sel = (int32_t *)(ws + sel_off);
        s.cand = (uint64_t *)(ws + cand_off);
        return s;
    }
};

DecodeLayout decode_layout(int B, int Hkv, int64_t Lc, int S, int topk) {
    DecodeLayout p;
    const int64_t Nc = Lc / S;
    const size_t pairs = (size_t)B * Hkv;
    p.pairs = (int64_t)pairs;
    p.splits = decode_splits(B, Hkv, Nc, num_sms());
    size_t off = decode_zero_head(B, Hkv);
    p.sel_off = off;
    off = align_up(off + sizeof(int32_t) * pairs * topk, 256);
    p.cand_off = off;
    off = align_up(off + sizeof(uint64_t) * pairs * p.splits * topk, 256);
    p.total = off;
    return p;
}

hsa_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? HSA_OK : HSA_ERR_CUDA; }

// Per-thread timing hook (hsa_set_stage_events).
constexpr int kMaxStageEvents = 8;
thread_local cudaEvent_t t_stage_events[kMaxStageEvents];
thread_local int t_n_stage_events = 0;
thread_local int t_launches = 0;      // kernels launched by this thread's last call

inline void stage_mark(int i, cudaStream_t st) {
    if (i < t_n_stage_events && t_stage_events[i]) cudaEventRecord(t_stage_events[i], st);
}
inline cudaEvent_t stage_event(int i) {
    return i < t_n_stage_events ? t_stage_events[i] : nullptr;
}

}  // namespace

extern "C" {

int hsa_version(void) { return 100; }

int hsa_last_call_launches(void) { return t_launches; }

unsigned hsa_last_call_kernels(void) { return t_kernels; }

hsa_status_t hsa_set_path_overrides(int flags, int64_t window_tokens) {
    const int known = HSA_PATH_SIMT_PREFILL | HSA_PATH_SIMT_SELECT | HSA_PATH_MULTI_TILE_SELECT;
    if ((flags & ~known) != 0 || window_tokens < 0 || (window_tokens > 0 && window_tokens < 256))
        return HSA_ERR_INVALID_ARG;
    t_path_flags = flags;
    t_window_tokens = window_tokens;
    return HSA_OK;
}

hsa_status_t hsa_set_stage_events(void *const *events, int n) {
    if (n < 0 || n > kMaxStageEvents || (n > 0 && !events)) return HSA_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i) t_stage_events[i] = (cudaEvent_t)events[i];
    t_n_stage_events = n;
    return HSA_OK;
}

const char *hsa_status_string(hsa_status_t s) {
    switch (s) {
    case HSA_OK: return "ok";
    case HSA_ERR_INVALID_ARG: return "invalid argument";
    case HSA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case HSA_ERR_WORKSPACE: return "workspace missing or too small";
    case HSA_ERR_CUDA: return "CUDA error";
    case HSA_ERR_TIMEOUT: return "device-side wait timed out";
    }
    return "unknown status";
}

hsa_status_t hsa_landmarks(const void *K, hsa_dtype_t k_dt, float *lm_out, int B, int Hkv,
                           int64_t L, int d, int S, void *stream) {
    hsa_status_t s = check_shape(B, Hkv, Hkv, L, d, S, 1);
    if (s != HSA_OK) return s;
    if (!dtype_ok(k_dt)) return HSA_ERR_UNSUPPORTED;
    t_launches = 0;
    t_kernels = 0;
    if (L / S == 0) return HSA_OK;
    if (!K || !lm_out || !aligned16(K) || !aligned16(lm_out)) return HSA_ERR_INVALID_ARG;
    t_launches = 1;
    t_kernels = HSA_K_LANDMARKS;
    return from_cuda(launch_landmarks(K, k_dt == HSA_BF16, lm_out, B, Hkv, L, d,
                                      (cudaStream_t)stream));
}

size_t hsa_prefill_workspace_size(int B, int H, int Hkv, int64_t L, int d, int S, int topk) {
    if (check_shape(B, H, Hkv, L, d, S, topk) != HSA_OK) return 0;
    return prefill_layout(B, H, Hkv, L, d, S, topk, L / S, false).total;
}

size_t hsa_prefill_varlen_workspace_size(int B, int H, int Hkv, int64_t L, int d, int64_t n_chunks,
                                         int topk) {
    if (check_shape(B, H, Hkv, L, d, kChunk, topk) != HSA_OK) return 0;
    if (n_chunks < 1 || n_chunks > L || n_chunks * (int64_t)kMaxVarChunk < L) return 0;
    return prefill_layout(B, H, Hkv, L, d, kChunk, topk, n_chunks, true).total;
}

hsa_status_t hsa_prefill(const void *Q, const void *K, const void *V, hsa_dtype_t dt,
                         const void *lm, hsa_dtype_t lm_dt, int B, int H, int Hkv, int64_t L,
                         int d, int S, int topk, int own_chunk, float scale, void *O,
                         int32_t *idx_out, float *w_out, void *workspace, size_t ws_bytes,
                         void *stream) {
    return hsa_prefill_variant(Q, K, V, dt, lm, lm_dt, B, H, Hkv, L, d, S, topk, own_chunk, scale,
                               nullptr, O, idx_out, w_out, workspace, ws_bytes, stream);
}

}  // extern "C"

namespace {

// The prefill behind every entry point: chunks of S tokens (bounds == null)
// or n_chunks variable-length chunks (bounds on the device).
hsa_status_t prefill_impl(const void *Q, const void *K, const void *V, hsa_dtype_t dt,
                          const void *lm, hsa_dtype_t lm_dt, int B, int H, int Hkv, int64_t L,
                          int d, int S, int topk, int own_chunk, float scale,
                          const hsa_variant_t *variant, const int32_t *bounds, int64_t n_chunks,
                          void *O, int32_t *idx_out, float *w_out, void *workspace,
                          size_t ws_bytes, void *stream) {
    hsa_status_t s = check_shape(B, H, Hkv, L, d, S, topk);
    if (s != HSA_OK) return s;
    const int R = variant ? variant->retrieval_interval : 1;
    const int pool_mean = variant ? variant->pool_mean : 0;
    const int union_softmax = variant ? variant->union_softmax : 0;
    if (R < 1 || S % R != 0 || (pool_mean != 0 && pool_mean != 1) ||
        (union_softmax != 0 && union_softmax != 1))
        return HSA_ERR_INVALID_ARG;
    if (!dtype_ok(dt) || !dtype_ok(lm_dt)) return HSA_ERR_UNSUPPORTED;
    if (own_chunk != 0 && own_chunk != 1) return HSA_ERR_INVALID_ARG;
    if (!(scale >= 0.f) || scale == INFINITY) return HSA_ERR_INVALID_ARG;
    t_launches = 0;
    t_kernels = 0;
    if (L == 0) return HSA_OK;
    const void *ptrs[] = {Q, K, V, O, workspace};
    for (const void *p : ptrs)
        if (!p || !aligned16(p)) return HSA_ERR_INVALID_ARG;
    if ((lm && !aligned16(lm)) || (idx_out && !aligned16(idx_out)) || (w_out && !aligned16(w_out)))
        return HSA_ERR_INVALID_ARG;
    const bool varlen = bounds != nullptr;
    const int64_t Nc = varlen ? n_chunks : L / S;
    const PrefillLayout lay = prefill_layout(B, H, Hkv, L, d, S, topk, Nc, varlen);
    if (ws_bytes < lay.total) return HSA_ERR_WORKSPACE;
    if (scale == 0.f) scale = 1.0f / sqrtf((float)d);

    cudaStream_t st = (cudaStream_t)stream;
    char *ws = (char *)workspace;
    int32_t *tok_chunk = varlen ? (int32_t *)(ws + lay.tokc_off) : nullptr;
    int32_t *idx = idx_out ? idx_out : (int32_t *)(ws + lay.idx_off);
    float *w = w_out ? w_out : (float *)(ws + lay.w_off);
    const bool bf16 = dt == HSA_BF16;
    const void *lm_use = lm;
    bool lm_bf16 = lm_dt == HSA_BF16;
    stage_mark(0, st);
    const bool use_tc = bf16 && lay.tc && !force_simt_path() &&
                        attend_tc_supported(bf16, H / Hkv, d);
    // the bucket counts are zeroed first, so that every kernel of the chain
    // can follow its predecessor as a programmatic dependent
    if (use_tc && cudaMemsetAsync(ws + lay.counts_off, 0, lay.counts_bytes, st) != cudaSuccess)
        return HSA_ERR_CUDA;
    if (varlen) {   // checked boundaries and the chunk of every token; every later
                    // kernel reads those (wrong boundaries flag the status word)
        int32_t *bs = (int32_t *)(ws + lay.bnds_off);
        if (launch_varlen_setup(bounds, n_chunks, L, bs, tok_chunk, (unsigned *)ws, st) !=
            cudaSuccess)
            return HSA_ERR_CUDA;
        t_launches += 2;
        bounds = bs;
    }
    if (!lm) {
        float *lm_ws = (float *)(ws + lay.lm_off);
        cudaError_t e = varlen ? launch_landmarks_varlen(K, bf16, lm_ws, B, Hkv, L, d, bounds,
                                                         n_chunks, st)
                               : launch_landmarks(K, bf16, lm_ws, B, Hkv, L, d, st);
        if (e != cudaSuccess) return HSA_ERR_CUDA;
        t_launches += Nc > 0 ? 1 : 0;
        t_kernels |= Nc > 0 ? (unsigned)HSA_K_LANDMARKS : 0u;
        lm_use = lm_ws;
        lm_bf16 = false;
    }
    stage_mark(1, st);
    // The tensor-core path computes the fusion logits inside its S tiles and
    // the weights in fuse_kernel, so the selection skips them there.
    cudaError_t e;
    // fp32 landmarks on the tensor-core path: split once into bf16 high / low
    // planes, which the selection and the attention tiles both read
    void *lm_split = ws + lay.lmsplit_off;
    if (use_tc && !lm_bf16 && Nc > 0) {
        e = launch_split_landmarks(lm_use, lm_split, (int64_t)B * Hkv * Nc * d, st);
        if (e != cudaSuccess) return HSA_ERR_CUDA;
        t_launches += 1;
        t_kernels |= HSA_K_SPLIT_LANDMARKS;
    }
    const bool tc_select = use_tc && Nc > 0 && (H / Hkv) % 8 == 0 && select_tc_supported() &&
                           !force_simt_select();
    bool multi = false;
    if (tc_select)
        e = launch_select_tc(Q, lm_use, lm_bf16, lm_split, B, H, Hkv, L, d, S, Nc, topk, scale, R,
                             pool_mean, bounds, tok_chunk, idx, (unsigned *)ws,
                             force_multi_tile_select(), &multi, st);
    else   // the CUDA-core attention takes the fusion weights from the selection
        e = launch_select(Q, bf16, lm_use, lm_bf16, B, H, Hkv, L, d, S, Nc, bounds, tok_chunk,
                          topk, scale, R, pool_mean, idx,
                          use_tc ? nullptr : (union_softmax ? (float *)(ws + lay.w_off) : w), st);
    if (e != cudaSuccess) return HSA_ERR_CUDA;
    t_launches += 1;
    t_kernels |= !tc_select ? HSA_K_SELECT_SIMT
                            : multi ? HSA_K_SELECT_TC_MULTI_TILE : HSA_K_SELECT_TC_ONE_TILE;
    stage_mark(2, st);
    if (use_tc) {
        e = launch_bucket(idx, B, Hkv, L, topk, Nc, S, bounds, tok_chunk, 128 / (H / Hkv), lay.W,
                          lay.cap, (int32_t *)(ws + lay.counts_off),
                          (int32_t *)(ws + lay.cursor_off), (int32_t *)(ws + lay.entries_off),
                          (int4 *)(ws + lay.wtiles_off), (int32_t *)(ws + lay.wntiles_off),
                          (int32_t *)(ws + lay.done_off), (int32_t *)(ws + lay.wown_off),
                          (int64_t *)(ws + lay.seg_off), (int4 *)(ws + lay.tiles_off), st);
        if (e != cudaSuccess) return HSA_ERR_CUDA;
        t_launches += 3;                  // count, scan, fill (scatter + flatten)
        t_kernels |= HSA_K_WORK_LISTS;
        stage_mark(3, st);
        TcLaunch a;
        a.Q = Q; a.K = K; a.V = V; a.lm = lm_bf16 ? lm_use : lm_split; a.lm_bf16 = lm_bf16 ? 1 : 0;
        a.B = B; a.H = H; a.Hkv = Hkv; a.S = S; a.topk = topk; a.own_chunk = own_chunk;
        a.L = L; a.W = lay.W; a.cap = lay.cap; a.scale = scale;
        a.idx = idx; a.entries = (const int32_t *)(ws + lay.entries_off);
        a.tiles = (const int4 *)(ws + lay.tiles_off);
        a.qlen = (const int64_t *)(ws + lay.seg_off) + 2 * lay.NW;
        a.zf = (float *)(ws + lay.zf_off); a.own_f = (float *)(ws + lay.ownf_off);
        a.own_m = (float *)(ws + lay.ownm_off); a.union_softmax = union_softmax;
        a.Nc = Nc; a.bounds = bounds; a.tok_chunk = tok_chunk;
        a.w_out = w_out;
        a.part = (__half *)(ws + lay.part_off); a.own = (__half *)(ws + lay.own_off);
        a.O = O; a.status = (unsigned *)ws;
        a.num_sms = num_sms();
        e = launch_attend_tc(a, d, st, stage_event(4));
        t_launches += e == cudaSuccess ? 2 : 0;
        t_kernels |= e == cudaSuccess ? (unsigned)(HSA_K_ATTEND_TC | HSA_K_FUSE) : 0u;
    } else {
        stage_mark(3, st);
        e = launch_attend_simt(Q, K, V, bf16, idx, union_softmax ? (float *)(ws + lay.w_off) : w,
                               B, H, Hkv, L, d, S, topk, own_chunk, scale, union_softmax, bounds,
                               tok_chunk, O, st);
        // the union softmax has no per-chunk fusion weights: w_out reads 0
        if (e == cudaSuccess && union_softmax && w_out)
            e = cudaMemsetAsync(w_out, 0, sizeof(float) * (size_t)B * L * H * topk, st);
        t_launches += e == cudaSuccess ? 1 : 0;
        t_kernels |= e == cudaSuccess ? (unsigned)HSA_K_ATTEND_SIMT : 0u;
        stage_mark(4, st);            // the SIMT kernel fuses in place
    }
    stage_mark(5, st);
    return from_cuda(e);
}

}  // namespace

extern "C" {

hsa_status_t hsa_prefill_variant(const void *Q, const void *K, const void *V, hsa_dtype_t dt,
                                 const void *lm, hsa_dtype_t lm_dt, int B, int H, int Hkv,
                                 int64_t L, int d, int S, int topk, int own_chunk, float scale,
                                 const hsa_variant_t *variant, void *O, int32_t *idx_out,
                                 float *w_out, void *workspace, size_t ws_bytes, void *stream) {
    return prefill_impl(Q, K, V, dt, lm, lm_dt, B, H, Hkv, L, d, S, topk, own_chunk, scale,
                        variant, nullptr, 0, O, idx_out, w_out, workspace, ws_bytes, stream);
}

hsa_status_t hsa_prefill_varlen(const void *Q, const void *K, const void *V, hsa_dtype_t dt,
                                const void *lm, hsa_dtype_t lm_dt, int B, int H, int Hkv,
                                int64_t L, int d, const int32_t *bounds, int64_t n_chunks,
                                int topk, int own_chunk, float scale, int union_softmax,
                                void *O, int32_t *idx_out, float *w_out, void *workspace,
                                size_t ws_bytes, void *stream) {
    if (n_chunks < 1 || n_chunks > L || n_chunks * (int64_t)kMaxVarChunk < L)
        return L == 0 ? HSA_OK : HSA_ERR_INVALID_ARG;
    if (!bounds || !aligned16(bounds)) return HSA_ERR_INVALID_ARG;
    const hsa_variant_t v = {1, 0, union_softmax};
    return prefill_impl(Q, K, V, dt, lm, lm_dt, B, H, Hkv, L, d, kChunk, topk, own_chunk, scale,
                        &v, bounds, n_chunks, O, idx_out, w_out, workspace, ws_bytes, stream);
}

size_t hsa_decode_workspace_size(int B, int H, int Hkv, int64_t Lc, int d, int S, int topk) {
    if (check_shape(B, H, Hkv, Lc, d, S, topk) != HSA_OK) return 0;
    if (Lc % S != 0) return 0;
    return decode_layout(B, Hkv, Lc, S, topk).total;
}

}  // extern "C"

namespace {

// hsa_decode and hsa_decode_ragged: lens = null, every sequence sees Lc tokens.
hsa_status_t decode_impl(const void *q, const void *Kc, const void *Vc, hsa_dtype_t dt,
                         const void *lm, hsa_dtype_t lm_dt, int B, int H, int Hkv, int64_t Lc,
                         int d, int S, int topk, float scale, const int32_t *lens, void *O,
                         int32_t *idx_out, void *workspace, size_t ws_bytes, void *stream) {
    hsa_status_t s = check_shape(B, H, Hkv, Lc, d, S, topk);
    if (s != HSA_OK) return s;
    if (!dtype_ok(dt) || !dtype_ok(lm_dt)) return HSA_ERR_UNSUPPORTED;
    if (Lc % S != 0) return HSA_ERR_INVALID_ARG;
    if (!(scale >= 0.f) || scale == INFINITY) return HSA_ERR_INVALID_ARG;
    t_launches = 0;
    t_kernels = 0;
    if (!q || !O || !workspace || !aligned16(q) || !aligned16(O) || !aligned16(workspace))
        return HSA_ERR_INVALID_ARG;
    if (idx_out && !aligned16(idx_out)) return HSA_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    if (Lc == 0) {   // nothing visible: O = 0, no selection
        const size_t el = dt == HSA_BF16 ? 2 : 4;
        if (cudaMemsetAsync(O, 0, el * (size_t)B * H * d, st) != cudaSuccess) return HSA_ERR_CUDA;
        if (idx_out && cudaMemsetAsync(idx_out, 0xff, sizeof(int32_t) * (size_t)B * Hkv * topk,
                                       st) != cudaSuccess)
            return HSA_ERR_CUDA;
        return HSA_OK;
    }
    const void *ptrs[] = {Kc, Vc, lm};
    for (const void *p : ptrs)
        if (!p || !aligned16(p)) return HSA_ERR_INVALID_ARG;
    const DecodeLayout lay = decode_layout(B, Hkv, Lc, S, topk);
    if (ws_bytes < lay.total) return HSA_ERR_WORKSPACE;
    if (scale == 0.f) scale = 1.0f / sqrtf((float)d);
    char *ws = (char *)workspace;
    stage_mark(0, st);
    DecodeShard whole = {0, nullptr, nullptr, nullptr, nullptr, nullptr};
    whole.lens = lens;
    whole.S = S;
    hsa_status_t r = from_cuda(launch_decode(q, Kc, Vc, dt == HSA_BF16, lm, lm_dt == HSA_BF16, B, H, Hkv,
                                   Lc, d, S, topk, scale, lay.splits, lay.at(ws), O,
                                   idx_out, whole, 0, nullptr, st));
    t_launches = r == HSA_OK ? 2 : 0;
    t_kernels = r == HSA_OK ? (unsigned)(HSA_K_DECODE_SCAN | HSA_K_DECODE_ATTEND) : 0u;
    stage_mark(1, st);
    return r;
}

}  // namespace

extern "C" {

hsa_status_t hsa_decode(const void *q, const void *Kc, const void *Vc, hsa_dtype_t dt,
                        const void *lm, hsa_dtype_t lm_dt, int B, int H, int Hkv, int64_t Lc,
                        int d, int S, int topk, float scale, void *O, int32_t *idx_out,
                        void *workspace, size_t ws_bytes, void *stream) {
    return decode_impl(q, Kc, Vc, dt, lm, lm_dt, B, H, Hkv, Lc, d, S, topk, scale, nullptr, O,
                       idx_out, workspace, ws_bytes, stream);
}

hsa_status_t hsa_decode_ragged(const void *q, const void *Kc, const void *Vc, hsa_dtype_t dt,
                               const void *lm, hsa_dtype_t lm_dt, int B, int H, int Hkv,
                               int64_t Lmax, int d, int S, int topk, float scale,
                               const int32_t *lens, void *O, int32_t *idx_out, void *workspace,
                               size_t ws_bytes, void *stream) {
    if (!lens || !aligned16(lens)) return HSA_ERR_INVALID_ARG;
    return decode_impl(q, Kc, Vc, dt, lm, lm_dt, B, H, Hkv, Lmax, d, S, topk, scale, lens, O,
                       idx_out, workspace, ws_bytes, stream);
}

hsa_status_t hsa_landmarks_append(const void *K, hsa_dtype_t k_dt, void *lm, hsa_dtype_t lm_dt,
                                  int B, int Hkv, int64_t Lmax, int d, int S,
                                  const int32_t *len_before, const int32_t *len_after,
                                  int max_new_chunks, void *stream) {
    hsa_status_t s = check_shape(B, Hkv, Hkv, Lmax, d, S, 1);
    if (s != HSA_OK) return s;
    if (!dtype_ok(k_dt) || !dtype_ok(lm_dt)) return HSA_ERR_UNSUPPORTED;
    if (Lmax % S != 0 || max_new_chunks < 0) return HSA_ERR_INVALID_ARG;
    t_launches = 0;
    t_kernels = 0;
    if (Lmax == 0) return HSA_OK;
    const void *ptrs[] = {K, lm, len_before, len_after};
    for (const void *p : ptrs)
        if (!p || !aligned16(p)) return HSA_ERR_INVALID_ARG;
    const cudaError_t e = launch_landmarks_append(K, k_dt == HSA_BF16, lm, lm_dt == HSA_BF16, B,
                                                  Hkv, Lmax, d, S, len_before, len_after,
                                                  max_new_chunks, (cudaStream_t)stream);
    if (e == cudaSuccess) {
        t_launches = 1;
        t_kernels = HSA_K_LANDMARKS;
    }
    return from_cuda(e);
}

hsa_status_t hsa_decode_cp_candidates(const void *q, hsa_dtype_t dt, const void *lm,
                                      hsa_dtype_t lm_dt, int B, int H, int Hkv, int64_t Lc, int d,
                                      int S, int topk, float scale, int64_t chunk_offset,
                                      float *cand_score, int32_t *cand_idx, void *workspace,
                                      size_t ws_bytes, void *stream) {
    hsa_status_t s = check_shape(B, H, Hkv, Lc, d, S, topk);
    if (s != HSA_OK) return s;
    if (!dtype_ok(dt) || !dtype_ok(lm_dt)) return HSA_ERR_UNSUPPORTED;
    if (Lc % S != 0 || chunk_offset < 0 || chunk_offset + Lc / S > (int64_t)INT32_MAX)
        return HSA_ERR_INVALID_ARG;
    if (!(scale >= 0.f) || scale == INFINITY) return HSA_ERR_INVALID_ARG;
    t_launches = 0;
    t_kernels = 0;
    const void *ptrs[] = {q, cand_score, cand_idx, workspace};
    for (const void *p : ptrs)
        if (!p || !aligned16(p)) return HSA_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    const size_t nc = (size_t)B * Hkv * topk;
    if (Lc == 0) {   // an empty shard has no candidates
        if (cudaMemsetAsync(cand_idx, 0xff, sizeof(int32_t) * nc, st) != cudaSuccess)
            return HSA_ERR_CUDA;
        return cudaMemsetAsync(cand_score, 0, sizeof(float) * nc, st) == cudaSuccess
                   ? HSA_OK : HSA_ERR_CUDA;
    }
    if (!lm || !aligned16(lm)) return HSA_ERR_INVALID_ARG;
    const DecodeLayout lay = decode_layout(B, Hkv, Lc, S, topk);
    if (ws_bytes < lay.total) return HSA_ERR_WORKSPACE;
    if (scale == 0.f) scale = 1.0f / sqrtf((float)d);
    const DecodeShard sh = {chunk_offset, cand_score, cand_idx, nullptr, nullptr, nullptr};
    const hsa_status_t r = from_cuda(launch_decode(q, nullptr, nullptr, dt == HSA_BF16, lm,
                                                   lm_dt == HSA_BF16, B, H, Hkv, Lc, d, S, topk,
                                                   scale, lay.splits, lay.at((char *)workspace),
                                                   nullptr, nullptr, sh, 1, nullptr, st));
    t_launches = r == HSA_OK ? 1 : 0;
    t_kernels = r == HSA_OK ? (unsigned)HSA_K_DECODE_SCAN : 0u;
    return r;
}

hsa_status_t hsa_decode_cp_merge(const float *cand_score, const int32_t *cand_idx, int R, int B,
                                 int Hkv, int topk, int32_t *idx, void *stream) {
    if (R < 1 || B < 1 || Hkv < 1 || topk < 1) return HSA_ERR_INVALID_ARG;
    if (topk > 32) return HSA_ERR_UNSUPPORTED;
    if (!cand_score || !cand_idx || !idx) return HSA_ERR_INVALID_ARG;
    t_launches = 0;
    t_kernels = 0;
    const hsa_status_t r = from_cuda(launch_decode_cp_merge(cand_score, cand_idx, R, B, Hkv, topk,
                                                            idx, (cudaStream_t)stream));
    t_launches = r == HSA_OK ? 1 : 0;
    t_kernels = r == HSA_OK ? (unsigned)HSA_K_DECODE_CP_MERGE : 0u;
    return r;
}

hsa_status_t hsa_decode_cp_attend(const void *q, const void *Kc, const void *Vc, hsa_dtype_t dt,
                                  const void *lm, hsa_dtype_t lm_dt, int B, int H, int Hkv,
                                  int64_t Lc, int d, int S, int topk, float scale,
                                  int64_t chunk_offset, const int32_t *idx, float *m, float *Z,
                                  float *acc, void *stream) {
    hsa_status_t s = check_shape(B, H, Hkv, Lc, d, S, topk);
    if (s != HSA_OK) return s;
    if (!dtype_ok(dt) || !dtype_ok(lm_dt)) return HSA_ERR_UNSUPPORTED;
    if (Lc % S != 0 || chunk_offset < 0 || chunk_offset + Lc / S > (int64_t)INT32_MAX)
        return HSA_ERR_INVALID_ARG;
    if (!(scale >= 0.f) || scale == INFINITY) return HSA_ERR_INVALID_ARG;
    t_launches = 0;
    t_kernels = 0;
    const void *ptrs[] = {q, idx, m, Z, acc};
    for (const void *p : ptrs)
        if (!p || !aligned16(p)) return HSA_ERR_INVALID_ARG;
    if (Lc > 0) {
        const void *cache[] = {Kc, Vc, lm};
        for (const void *p : cache)
            if (!p || !aligned16(p)) return HSA_ERR_INVALID_ARG;
    }
    if (scale == 0.f) scale = 1.0f / sqrtf((float)d);
    const DecodeShard sh = {chunk_offset, nullptr, nullptr, m, Z, acc};
    DecodeScratch none = {nullptr, nullptr, nullptr, nullptr, nullptr};
    const hsa_status_t r = from_cuda(launch_decode(q, Kc, Vc, dt == HSA_BF16, lm,
                                                   lm_dt == HSA_BF16, B, H, Hkv, Lc, d, S, topk,
                                                   scale, 1, none, nullptr, nullptr, sh, 2, idx,
                                                   (cudaStream_t)stream));
    t_launches = r == HSA_OK ? 1 : 0;
    t_kernels = r == HSA_OK ? (unsigned)HSA_K_DECODE_ATTEND : 0u;
    return r;
}

hsa_status_t hsa_decode_cp_combine(const float *m, const float *Z, const float *acc, int R, int B,
                                   int H, int d, hsa_dtype_t dt, void *O, void *stream) {
    if (R < 1 || B < 1 || H < 1 || d < 1) return HSA_ERR_INVALID_ARG;
    if (!dtype_ok(dt)) return HSA_ERR_UNSUPPORTED;
    if (!m || !Z || !acc || !O || !aligned16(O)) return HSA_ERR_INVALID_ARG;
    t_launches = 0;
    t_kernels = 0;
    const hsa_status_t r = from_cuda(launch_decode_cp_combine(m, Z, acc, R, B, H, d,
                                                              dt == HSA_BF16, O,
                                                              (cudaStream_t)stream));
    t_launches = r == HSA_OK ? 1 : 0;
    t_kernels = r == HSA_OK ? (unsigned)HSA_K_DECODE_CP_COMBINE : 0u;
    return r;
}

hsa_status_t hsa_selftest_wait_expiry(void *workspace, size_t ws_bytes, int64_t budget_cycles,
                                      void *stream) {
    if (budget_cycles < 1 || budget_cycles > 4000000000LL) return HSA_ERR_INVALID_ARG;
    if (!workspace) {
        // aimed at the status word of hsa_decode_noalloc's array on the stream's device
        const hsa_status_t s = noalloc_status_word((cudaStream_t)stream, true, &workspace);
        if (s != HSA_OK) return s;
        ws_bytes = kStatusBytes;
    }
    if (ws_bytes < 16 || ((uintptr_t)workspace & 15) != 0) return HSA_ERR_INVALID_ARG;
    return hsa::launch_selftest_wait((unsigned *)workspace, (long long)budget_cycles,
                                     (cudaStream_t)stream) == cudaSuccess ? HSA_OK : HSA_ERR_CUDA;
}

size_t hsa_prefill_backward_workspace_size(int B, int H, int Hkv, int64_t L, int d, int S,
                                           int topk, int dhsa) {
    if (check_shape(B, H, Hkv, L, d, S, topk) != HSA_OK) return 0;
    if (L >= ((int64_t)1 << 26) || (int64_t)B * Hkv * L * topk >= (int64_t)INT32_MAX) return 0;
    // room for the tensor-core path whenever the shape could take it (bf16 inputs)
    return bwd_layout(B, H, Hkv, L, d, S, topk, dhsa != 0, H / Hkv == 8 && d == 128).total;
}

hsa_status_t hsa_prefill_backward(const void *Q, const void *K, const void *V, hsa_dtype_t dt,
                                  const void *lm, hsa_dtype_t lm_dt, const int32_t *idx,
                                  const void *dO, int B, int H, int Hkv, int64_t L, int d, int S,
                                  int topk, int own_chunk, float scale, float *dQ, float *dK,
                                  float *dV, float *dlm, void *workspace, size_t ws_bytes,
                                  void *stream) {
    hsa_status_t s = check_shape(B, H, Hkv, L, d, S, topk);
    if (s != HSA_OK) return s;
    if (!dtype_ok(dt) || !dtype_ok(lm_dt)) return HSA_ERR_UNSUPPORTED;
    if (own_chunk != 0 && own_chunk != 1) return HSA_ERR_INVALID_ARG;
    if (!(scale >= 0.f) || scale == INFINITY) return HSA_ERR_INVALID_ARG;
    // entry codes t*32 + slot and entry offsets are 32-bit
    if (L >= ((int64_t)1 << 26) || (int64_t)B * Hkv * L * topk >= (int64_t)INT32_MAX)
        return HSA_ERR_UNSUPPORTED;
    t_launches = 0;
    t_kernels = 0;
    if (L == 0) return HSA_OK;
    const void *ptrs[] = {Q, K, V, dO, idx, dQ, dK, dV, workspace};
    for (const void *p : ptrs)
        if (!p || !aligned16(p)) return HSA_ERR_INVALID_ARG;
    const bool dhsa = lm == nullptr;
    if (!dhsa && (!aligned16(lm) || !dlm || !aligned16(dlm))) return HSA_ERR_INVALID_ARG;
    const bool tc = backward_tc_supported(dt == HSA_BF16, H / Hkv, d) && !force_simt_path();
    const BwdLayout lay = bwd_layout(B, H, Hkv, L, d, S, topk, dhsa, tc);
    if (ws_bytes < lay.total) return HSA_ERR_WORKSPACE;
    if (scale == 0.f) scale = 1.0f / sqrtf((float)d);
    cudaStream_t st = (cudaStream_t)stream;
    char *ws = (char *)workspace;
    BwdArgs a;
    a.Q = Q; a.K = K; a.V = V; a.dO = dO; a.lm = lm;
    a.lm_bf16 = lm_dt == HSA_BF16; a.bf16 = dt == HSA_BF16; a.dhsa = dhsa;
    a.idx = idx; a.B = B; a.H = H; a.Hkv = Hkv; a.d = d; a.S = S; a.topk = topk;
    a.own_chunk = own_chunk; a.L = L; a.scale = scale;
    a.dQ = dQ; a.dK = dK; a.dV = dV; a.dlm = dhsa ? nullptr : dlm; a.ws = workspace;
    stage_mark(0, st);
    if (dhsa) {   // the landmarks the forward used: sqrt(S) * mean of each chunk's keys
        float *lm_ws = (float *)(ws + lay.lm_off);
        if (lay.Nc > 0) {
            if (launch_landmarks(K, a.bf16, lm_ws, B, Hkv, L, d, st) != cudaSuccess)
                return HSA_ERR_CUDA;
            t_launches += 1;
            t_kernels |= HSA_K_LANDMARKS;
        }
        a.lm = lm_ws;
        a.lm_bf16 = 0;
    }
    const cudaError_t e = launch_backward(a, lay, st);
    if (e == cudaSuccess) {
        // CUDA cores: row, [hist], scan, [scatter], key, reduce; tensor cores: weights,
        // [hist], scan, [scatter], key (tcgen05), row finish, dl, reduce
        t_launches += (tc ? 6 : 4) + (lay.Nc > 0 ? 2 : 0);
        t_kernels |= HSA_K_BACKWARD | (tc ? (unsigned)HSA_K_BACKWARD_TC : 0u);
    }
    stage_mark(1, st);
    return from_cuda(e);
}

hsa_status_t hsa_check(void *workspace, void *stream) {
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return HSA_ERR_CUDA;
    if (!workspace) {
        // Calls without a workspace (hsa_decode_noalloc) flag the status word
        // at the head of the library's array on the stream's device.
        if (noalloc_status_word((cudaStream_t)stream, false, &workspace) != HSA_OK)
            return HSA_ERR_CUDA;
        if (!workspace) return HSA_OK;
    }
    unsigned flags = 0;
    if (cudaMemcpy(&flags, workspace, sizeof(flags), cudaMemcpyDeviceToHost) != cudaSuccess)
        return HSA_ERR_CUDA;
    if (flags & (kFlagTimeout | kFlagBadBounds | kFlagBadIdx)) {
        const unsigned zero = 0;
        cudaMemcpy(workspace, &zero, sizeof(zero), cudaMemcpyHostToDevice);
        return (flags & kFlagTimeout) ? HSA_ERR_TIMEOUT : HSA_ERR_INVALID_ARG;
    }
    return HSA_OK;
}

}  // extern "C"
