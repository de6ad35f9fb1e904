// scan_noalloc.cu -- ssd_chunk_scan_noalloc: ssd_chunk_scan with its
// workspace (the balanced schedule's hand-off slots and flags) taken from a
// static device array of the library instead of from the caller.
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/ssm.h"

// The scratch: SSM_NOALLOC_SCRATCH_BYTES of device memory per device,
// reserved when the library's device code is loaded on that device.
static __device__ __align__(256) unsigned char g_scratch[SSM_NOALLOC_SCRATCH_BYTES];

namespace {

// Its device address on each device, looked up on the first call made on
// that device (any thread may do the lookup; they all store the same value).
constexpr int kMaxDevices = 64;
std::atomic<void *> g_scratch_addr[kMaxDevices];

int scratch_of_current_device(void **addr)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SSM_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return SSM_ERR_UNSUPPORTED;
    void *p = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (!p) {
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return SSM_ERR_CUDA;
        g_scratch_addr[dev].store(p, std::memory_order_release);
    }
    *addr = p;
    return SSM_OK;
}

}  // namespace

extern "C" SSM_API int ssd_chunk_scan_noalloc(int nseq, int seqlen, const int32_t *cu_seqlens,
                                              int nheads, int head_dim, int d_state, int ngroups,
                                              int chunk_size, int in_dtype,
                                              const void *x, const float *dt, const float *A,
                                              const void *B, const void *C, const float *D,
                                              const float *initial_state,
                                              int y_dtype, void *y, float *final_state,
                                              int *status_dev, cudaStream_t stream)
{
    // Packed varlen input never uses a workspace; fixed-length shapes use
    // the one ssd_chunk_scan_workspace_size names (0 when none helps).
    const size_t need = cu_seqlens ? 0
                                   : ssd_chunk_scan_workspace_size(nseq, seqlen, nheads, head_dim,
                                                                   d_state, ngroups, chunk_size);
    if (need > SSM_NOALLOC_SCRATCH_BYTES) return SSM_ERR_SCRATCH_LIMIT;
    void *scratch = nullptr;
    if (need) {
        const int st = scratch_of_current_device(&scratch);
        if (st != SSM_OK) return st;
    }
    return ssd_chunk_scan(nseq, seqlen, cu_seqlens, nheads, head_dim, d_state, ngroups, chunk_size,
                          in_dtype, x, dt, A, B, C, D, initial_state, y_dtype, y, final_state,
                          scratch, need, status_dev, stream);
}
