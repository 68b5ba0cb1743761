// noalloc.cu — ca_chunk_attention_noalloc: the chunk attention call for callers
// that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocator) at the point where they
// run attention: an engine whose memory is carved up once at start-up and may
// not grow, code running inside a pre-sized memory pool, or a host path that
// must not take the allocator's locks. ca_chunk_attention needs a caller-owned
// workspace; this variant uses a fixed scratch array that lives in the library
// instead, so the caller passes only inputs and outputs.
//
// The scratch is a file-scope __device__ array: every GPU that loads the library
// holds kNoAllocScratchBytes of it until the process exits. Host code cannot use
// the array's name as a device address (on the host it is only a stand-in), so
// the first call on each device looks the address up with cudaGetSymbolAddress,
// with that device current, and keeps it.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "ca_internal.h"

namespace {

// Size of the library's scratch array. The attention kernels need a 256-byte
// header (the device status word) at minimum; the partial results of the
// last-wave split need far more, so the kernels, seeing a workspace this
// small, run unsplit.
constexpr size_t kNoAllocScratchBytes = 4096;
static_assert(kNoAllocScratchBytes >= ca::kWorkspaceHeader, "scratch below the minimum");
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char ca_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_setup_mutex;
void *g_scratch[kMaxDevices] = {nullptr};

// Device address of this device's scratch array (looked up once per device).
int scratch_for_current_device(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_scratch[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, ca_noalloc_scratch) != cudaSuccess || p == nullptr)
            return CA_ERR_CUDA;
        g_scratch[dev] = p;
    }
    *out = g_scratch[dev];
    return CA_OK;
}

}  // namespace

extern "C" int ca_chunk_attention_noalloc(const void *Q, const void *K, const void *V,
                                          const int32_t *tables, const int32_t *counts,
                                          const int32_t *chunk_start, int B, int H_q, int H_kv,
                                          int C, int L_max, int D, int blk, float scale, void *O,
                                          float *LSE, unsigned int *device_status, void *stream) {
    // The same host checks (and error codes) as ca_chunk_attention, before
    // anything is enqueued, so that a rejected call leaves the status word of
    // calls still in flight alone. The checks only test the workspace
    // pointer's alignment and size, so a 256-aligned placeholder stands in
    // for the scratch array here (it is never dereferenced).
    const int chk = ca::check_attention(Q, K, V, tables, counts, false, chunk_start, B, H_q, H_kv,
                                        C, L_max, D, blk, scale, O, LSE,
                                        reinterpret_cast<const void *>(uintptr_t{256}),
                                        kNoAllocScratchBytes);
    if (chk != CA_OK) return chk;
    void *scratch = nullptr;
    const int st = scratch_for_current_device(&scratch);
    if (st != CA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // The array keeps the previous call's contents; the status word must start
    // at zero for this call.
    if (cudaMemsetAsync(scratch, 0, sizeof(unsigned int), s) != cudaSuccess) return CA_ERR_CUDA;
    const int rc = ca_chunk_attention(Q, K, V, tables, counts, chunk_start, B, H_q, H_kv, C,
                                      L_max, D, blk, scale, O, LSE, scratch, kNoAllocScratchBytes,
                                      stream);
    if (rc != CA_OK) return rc;
    if (device_status != nullptr &&
        cudaMemcpyAsync(device_status, scratch, sizeof(unsigned int), cudaMemcpyDeviceToDevice,
                        s) != cudaSuccess)
        return CA_ERR_CUDA;
    return CA_OK;
}
