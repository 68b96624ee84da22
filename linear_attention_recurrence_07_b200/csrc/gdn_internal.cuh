// Internal declarations shared by the kernels and the C-ABI layer of libgdn.so.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "gdn.h"

namespace gdn {

constexpr int kHeadDim = 128;   // dk == dv == 128: the head size of the model (section 2.1)
constexpr int kChunk = 64;      // tokens per chunk of the chunkwise form

// Kernel arguments of the chunked prefill (plain pointers; shapes validated by the caller).
struct ChunkArgs {
    const void *q, *k, *v;
    const float *alpha, *beta, *S0;
    void *o;
    float *S_final;
    int B, T, Hqk, Hv;
    // Packed sequences: B sequences at token rows cu_seqlens[b] .. cu_seqlens[b+1]
    // of token arrays with one batch row of T tokens; null for [B, T, ...] arrays.
    const int *cu_seqlens = nullptr;
};

struct DecodeArgs {
    const void *q, *k, *v;
    const float *alpha, *beta, *S;
    void *o;
    float *S_new;
    int B, Hqk, Hv;
    int ntok = 1;                // tokens per sequence
    float *S_steps = nullptr;    // state after each token, or null
    const int *slots = nullptr;  // pool index of each sequence's state, or null
    int n_slots = 0;
};

// Launchers: enqueue on `stream`, return the launch's cudaError_t.
cudaError_t launch_decode(const DecodeArgs &a, gdn_dtype dtype, cudaStream_t stream);
cudaError_t launch_chunk_simt(const ChunkArgs &a, gdn_dtype dtype, cudaStream_t stream);
cudaError_t launch_chunk_tc(const ChunkArgs &a, cudaStream_t stream);
bool chunk_tc_available();
// Segment-parallel prefill (bf16, tensor cores): each sequence in up to `segments`
// pieces; workspace of chunk_tc_split_workspace bytes (0: no split needed).
size_t chunk_tc_split_workspace(int B, int T, int Hv, int segments);
cudaError_t launch_chunk_tc_split(const ChunkArgs &a, int segments, void *workspace,
                                  cudaStream_t stream);
// Scratch gdn_chunk_fwd_split uses for these arguments (0: it will not split).
size_t split_scratch_needed(int B, int T, int Hv, int dk, int dv, int segments, gdn_dtype dtype);
// Backward pass (gdn_bwd.cu): gradients of q, k, v, alpha, beta, S0.
struct BwdLaunch {
    const void *q, *k, *v, *dO;
    const float *alpha, *beta, *S0, *dS_final;
    float *dq, *dk, *dv, *dalpha, *dbeta, *dS0;
    float *work;
    int B, T, Hqk, Hv;
};
size_t bwd_workspace(int B, int T, int Hv);
cudaError_t launch_bwd(const BwdLaunch &L, gdn_dtype dtype, cudaStream_t stream);
// Chunkwise backward (gdn_bwd_chunk.cu, bf16 inputs): prep, forward state chain,
// gradient chain and per-chunk gradients; workspace of bwd_chunk_workspace bytes.
size_t bwd_chunk_workspace(int B, int T, int Hv);
cudaError_t launch_bwd_chunk(const BwdLaunch &L, cudaStream_t stream);

// Pipelined prefill (gdn_chunk_pipe.cu): prep CTAs stream each chunk's WY operands
// to state-carrying chain CTAs through a ring in the workspace (cooperative launch).
int chunk_pipe_chain_ctas(int B, int Hqk, int Hv, int sms, int req);
size_t chunk_pipe_workspace(int B, int Hqk, int Hv);
cudaError_t launch_chunk_pipe(const ChunkArgs &a, int chain_ctas, long long wait_limit,
                              void *workspace, size_t workspace_bytes, cudaStream_t stream);
// Read and clear a kernel file's device error word (bit 0: a bounded wait gave up).
cudaError_t chunk_pipe_take_error(unsigned *out);
cudaError_t chunk_tc_take_error(unsigned *out);
cudaError_t split_take_error(unsigned *out);

// sst: null, or where the first segments write S_start(1)^T in bf16 (see TcParams).
cudaError_t launch_chunk_tc_segments(const ChunkArgs &a, int seg_len, int nseg, float *segD,
                                     float *segM, __nv_bfloat16 *R, __nv_bfloat16 *sst,
                                     cudaStream_t stream);

// Element conversions used by the kernels.
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// log(alpha) with the documented clamp, so alpha == 0 stays finite.
__device__ __forceinline__ float clamped_log(float alpha) {
    return fmaxf(logf(alpha), -87.0f);
}

}  // namespace gdn
