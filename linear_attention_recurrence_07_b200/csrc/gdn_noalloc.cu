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
#include "gdn_internal.cuh"

namespace {

constexpr size_t kStaticScratchBytes = size_t(48) << 20;   // 48 MiB

static __device__ __align__(256) unsigned char g_split_scratch[kStaticScratchBytes];

// Device address of the array in the current device's context.  Looked up on every
// call (cheap once the module is loaded), so it is never stale: after a context is
// torn down and created again (cudaDeviceReset), the module and its array may sit
// at another address.
cudaError_t scratch_address(void **out)
{
    return cudaGetSymbolAddress(out, g_split_scratch);
}

}  // namespace

extern "C" gdn_status gdn_chunk_fwd_split_noalloc(const void *q, const void *k, const void *v,
                                                  const float *alpha, const float *beta,
                                                  const float *S0, void *o, float *S_final,
                                                  int B, int T, int Hqk, int Hv, int dk, int dv,
                                                  int chunk, int segments, gdn_dtype dtype,
                                                  void *stream)
{
    // the scratch the split itself will use (0 when it goes straight to gdn_chunk_fwd)
    const size_t need = gdn::split_scratch_needed(B, T, Hv, dk, dv, segments, dtype);
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
