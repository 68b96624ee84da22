// gdn_chunk_fwd_split_noalloc: the segment-parallel prefill with its scratch in a
// static device array, for callers that cannot allocate device memory.
//
// Some callers have no way to hand the library device memory: a host program
// whose device memory belongs to a pool it may not grow, or code that runs while
// allocation is forbidden (for instance between the steps of a memory plan fixed
// ahead of time).  gdn_chunk_fwd_split needs a workspace; this entry point uses a
// file-scope array of kStaticScratchBytes instead and calls nothing that
// allocates.  Every call shares that one array, so calls that overlap on the GPU
// race; nothing in it has to start at zero (every byte the split reads was written
// earlier in the same call).
#include <mutex>

#include "gdn_internal.cuh"

namespace {

constexpr size_t kStaticScratchBytes = size_t(48) << 20;   // 48 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_split_scratch[kStaticScratchBytes];

std::mutex g_scratch_mutex;
void *g_scratch_addr[kMaxDevices];   // device address of g_split_scratch, per device

// Address of the array on the current device: looked up once per device.
cudaError_t scratch_address(void **out)
{
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        err = cudaGetSymbolAddress(&p, g_split_scratch);
        if (err != cudaSuccess) return err;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" gdn_status gdn_chunk_fwd_split_noalloc(const void *q, const void *k, const void *v,
                                                  const float *alpha, const float *beta,
                                                  const float *S0, void *o, float *S_final,
                                                  int B, int T, int Hqk, int Hv, int dk, int dv,
                                                  int chunk, int segments, gdn_dtype dtype,
                                                  void *stream)
{
    // only bf16 calls split (and need scratch); the others go straight through
    const size_t need = dtype == GDN_BF16 ? gdn_chunk_fwd_split_workspace(B, T, Hv, dk, dv, segments) : 0;
    if (need > kStaticScratchBytes) return GDN_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    if (need > 0) {
        const cudaError_t err = scratch_address(&scratch);
        if (err != cudaSuccess) {
            cudaGetLastError();
            return GDN_ERR_CUDA;
        }
    }
    return gdn_chunk_fwd_split(q, k, v, alpha, beta, S0, o, S_final, B, T, Hqk, Hv, dk, dv, chunk,
                               segments, dtype, scratch, kStaticScratchBytes, stream);
}
