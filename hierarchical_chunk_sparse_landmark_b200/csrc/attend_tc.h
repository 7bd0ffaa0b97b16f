// attend_tc.h -- host-side launch interface of the tensor-core prefill
// attention (attend_tc.cu), shared with the C-ABI dispatch (abi.cu).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace hsa {

struct TcLaunch {
    const void *Q, *K, *V;
    // landmarks as bf16 rows: [B*Hkv*Nc, D] (lm_bf16) or the two planes
    // [2][B*Hkv*Nc, D] of an fp32 landmark's bf16 high and low parts
    const void *lm;
    int B, H, Hkv, S, topk, own_chunk, lm_bf16;
    int64_t L, W, cap;
    float scale;
    const int32_t *idx, *entries;
    const int4 *tiles;                // one descriptor per queue position
    const int64_t *qlen;              // number of tiles (device)
    float *zf, *own_f, *w_out;        // zf: [B, L, H, topk] float2; own_f: [B, L, H]
    float *own_m;                     // [B, L, H]: own-chunk row max (union softmax)
    int union_softmax;                // 1: one softmax over the union of the selected keys
    int64_t Nc;                       // chunks with a landmark
    const int32_t *bounds, *tok_chunk;  // variable-length chunks (null: chunks of S tokens)
    __half *part, *own;              // fp16 chunk outputs / own-chunk term
    void *O;
    unsigned *status;
    int num_sms;
};

bool attend_tc_supported(bool bf16, int G, int d);
int64_t attend_tc_max_windows();
// `mid` (may be null) is recorded between the attention and fusion kernels.
cudaError_t launch_attend_tc(const TcLaunch &a, int d, cudaStream_t st, cudaEvent_t mid);

}  // namespace hsa
