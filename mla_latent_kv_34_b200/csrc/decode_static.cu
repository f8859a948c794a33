// mla_decode_static: the decode step with library-owned scratch.
//
// Some callers cannot allocate device memory at the point where they decode:
// a runtime whose allocator is frozen once its memory pools are carved out,
// a host thread that must not enter the CUDA allocator (it can synchronise
// the device), or code that owns no torch or CUDA allocator at all.  For
// them this entry point takes no workspace argument; the segment partials go
// to one fixed buffer compiled into the library as a __device__ array, and
// nothing on this path calls cudaMalloc, cudaFree or any allocating library.
//
// Limits and rules, also stated in mla.h:
//  * the buffer holds MLA_DECODE_STATIC_SCRATCH_BYTES; a shape whose
//    mla_decode_workspace_bytes() exceeds it is rejected with
//    MLA_ERR_WORKSPACE before anything is launched;
//  * nothing in the buffer has to start at zero: every partial that the
//    finish phase reads is written by the attend phase of the same call;
//  * the first call on a device looks the buffer's address up (this can load
//    the library's device code on that device), so make it once before any
//    stream capture;
//  * there is one buffer per device, so calls that may overlap on the same
//    device (different streams, or different host threads without ordering)
//    race on it; calls ordered on one stream do not.
#include <stdint.h>

#include <mutex>

#include "mla_internal.cuh"

namespace {

__device__ __align__(256) unsigned char g_decode_scratch[MLA_DECODE_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Address of this device's scratch; the lookup runs once per device.
cudaError_t scratch_for_current_device(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess) return e;
        if (!p || (reinterpret_cast<uintptr_t>(p) & 255u) != 0) return cudaErrorInvalidDevicePointer;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" mla_status mla_decode_static(const void* q, const void* cache, int64_t cap_blocks,
                                        const int32_t* block_table, int max_blocks, const int32_t* kv_len,
                                        const void* W_UV, int B,
                                        int n_q, int H, float scale, int num_splits, void* out, float* lse_out,
                                        int32_t* dev_status, mla_stream stream) {
    if (B < 0 || n_q < 1 || H < 1 || num_splits < 0) return MLA_ERR_INVALID_ARG;
    const size_t need = mla_decode_workspace_bytes(B, n_q, H, num_splits);
    if (need > static_cast<size_t>(MLA_DECODE_STATIC_SCRATCH_BYTES)) return MLA_ERR_WORKSPACE;
    if (B == 0) return MLA_OK;
    // argument errors are reported before the device is touched, as for every other entry point
    if (!q || !cache || !block_table || !kv_len || !W_UV || !out) return MLA_ERR_INVALID_ARG;
    void* scratch = nullptr;
    if (scratch_for_current_device(&scratch) != cudaSuccess) return MLA_ERR_CUDA;
    return mla_decode(q, cache, cap_blocks, block_table, max_blocks, kv_len, W_UV, B, n_q, H, scale, num_splits, scratch,
                      static_cast<size_t>(MLA_DECODE_STATIC_SCRATCH_BYTES), out, lse_out, dev_status, stream);
}
