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
// library holds it until the process exits.  Host code cannot use the
// array's name as a device address (on the host it names a stand-in), so the
// device address is looked up with cudaGetSymbolAddress, with the stream's
// device current, and handed to the kernels.  The lookup is repeated on every
// call (a hash lookup once the module is loaded), so an address never
// outlives a cudaDeviceReset.
//
// The array's first 256 bytes are a status word like a workspace's: a
// kernel whose bounded wait runs out sets a flag there; the flag stays set
// across calls until hsa_check(NULL, stream) reports and clears it.
#include <atomic>

#include "common.cuh"
#include "hsa.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;     // 1 MiB per device

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 128;
std::atomic<bool> g_used[kMaxDevices];       // zero-initialised (static storage)

// Device of `stream` (the current device for the legacy default stream).
hsa_status_t stream_device(cudaStream_t stream, int *dev) {
    if (cudaStreamGetDevice(stream, dev) != cudaSuccess && cudaGetDevice(dev) != cudaSuccess)
        return HSA_ERR_CUDA;
    if (*dev < 0 || *dev >= kMaxDevices) return HSA_ERR_UNSUPPORTED;
    return HSA_OK;
}

// Device address of g_decode_scratch on device `dev`, looked up with that
// device current (the caller's current device is restored).
hsa_status_t scratch_address_on(int dev, void **out) {
    int cur = 0;
    if (cudaGetDevice(&cur) != cudaSuccess) return HSA_ERR_CUDA;
    if (cur != dev && cudaSetDevice(dev) != cudaSuccess) return HSA_ERR_CUDA;
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (cur != dev) cudaSetDevice(cur);
    if (e != cudaSuccess || p == nullptr) return HSA_ERR_CUDA;
    *out = p;
    return HSA_OK;
}

}  // namespace

namespace hsa {

// The status word of the array on `stream`'s device, for hsa_check and the
// self-test: *out = nullptr when nothing in this process has used the array
// on that device (unless `mark`, which records a use first).
hsa_status_t noalloc_status_word(cudaStream_t stream, bool mark, void **out) {
    *out = nullptr;
    int dev = 0;
    const hsa_status_t s = stream_device(stream, &dev);
    if (s != HSA_OK) return s;
    if (mark) g_used[dev].store(true, std::memory_order_relaxed);
    if (!g_used[dev].load(std::memory_order_relaxed)) return HSA_OK;
    return scratch_address_on(dev, out);
}

}  // namespace hsa

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
    const cudaStream_t st = (cudaStream_t)stream;
    int dev = 0;
    hsa_status_t s = stream_device(st, &dev);
    if (s != HSA_OK) return s;
    void *scratch = nullptr;
    s = scratch_address_on(dev, &scratch);
    if (s != HSA_OK) return s;
    g_used[dev].store(true, std::memory_order_relaxed);
    {
        // The tickets and the work counters (the head of the decode scratch
        // after the status word) must start at zero; the rest is fully
        // rewritten by every call.  The array keeps the previous call's
        // contents, so they are cleared here, on the caller's stream.  The
        // status word is left alone: a timeout flag stays until hsa_check
        // reports it.
        const size_t head = hsa::decode_zero_head(B, Hkv);
        const size_t clear = (head < need ? head : need) - hsa::kStatusBytes;
        if (cudaMemsetAsync((char *)scratch + hsa::kStatusBytes, 0, clear, st) != cudaSuccess)
            return HSA_ERR_CUDA;
    }
    return hsa_decode(q, Kc, Vc, dt, lm, lm_dt, B, H, Hkv, Lc, d, S, topk, scale, O, idx_out,
                      scratch, kNoAllocScratchBytes, stream);
}
