// decode_noalloc.cu -- hsa_decode_noalloc: the decode of hsa_decode for
// callers that cannot allocate device memory.
//
// Who needs it: code that runs inside a host program which owns all device
// memory (a serving engine that reserves the whole HBM for its KV cache at
// start-up, or a plugin interface that hands over only the input and output
// buffers), and code on a latency-critical path that must not call
// cudaMalloc/cudaFree because they can synchronise the device.  Such a caller
// cannot provide the workspace hsa_decode asks for.
//
// What it does instead: the decode scratch (per-(sequence, KV group) tickets
// and work counters, candidate lists and the selection) lives in one
// fixed-size array in device global memory that belongs to this library.
// The array is declared at file scope below, so every GPU that loads the
// library holds it until the process exits.  Host code cannot use the array's name as a device address (on the
// host it names a stand-in), so the device address is looked up once per
// device with cudaGetSymbolAddress and handed to the kernel.
#include <mutex>

#include "common.cuh"
#include "hsa.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;     // 1 MiB per device

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 128;
std::mutex g_scratch_mu;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device (looked up on the
// first call per device, with that device current).
hsa_status_t scratch_address(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return HSA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return HSA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess || p == nullptr) return HSA_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return HSA_OK;
}

}  // namespace

extern "C" size_t hsa_decode_noalloc_max_scratch(void) { return kNoAllocScratchBytes; }

extern "C" hsa_status_t hsa_decode_noalloc(const void *q, const void *Kc, const void *Vc,
                                           hsa_dtype_t dt, const void *lm, hsa_dtype_t lm_dt,
                                           int B, int H, int Hkv, int64_t Lc, int d, int S,
                                           int topk, float scale, void *O, int32_t *idx_out,
                                           void *stream) {
    const size_t need = hsa_decode_workspace_size(B, H, Hkv, Lc, d, S, topk);
    if (need == 0)   // invalid arguments: let hsa_decode report which, launching nothing
        return hsa_decode(q, Kc, Vc, dt, lm, lm_dt, B, H, Hkv, Lc, d, S, topk, scale, O, idx_out,
                          nullptr, 0, stream);
    if (need > kNoAllocScratchBytes) return HSA_ERR_WORKSPACE;   // beyond the fixed array
    void *scratch = nullptr;
    const hsa_status_t s = scratch_address(&scratch);
    if (s != HSA_OK) return s;
    {
        // The status word, the tickets and the work counters (the head of the
        // decode scratch) must start at zero; the rest is fully rewritten by
        // every call.  The array keeps the previous call's contents, so the
        // head is cleared here, on the caller's stream.
        const size_t head = hsa::decode_zero_head(B, Hkv);
        const size_t clear = head < need ? head : need;
        if (cudaMemsetAsync(scratch, 0, clear, (cudaStream_t)stream) != cudaSuccess)
            return HSA_ERR_CUDA;
    }
    return hsa_decode(q, Kc, Vc, dt, lm, lm_dt, B, H, Hkv, Lc, d, S, topk, scale, O, idx_out,
                      scratch, kNoAllocScratchBytes, stream);
}
