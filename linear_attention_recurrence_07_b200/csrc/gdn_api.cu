// C ABI of libgdn.so: argument checks and dispatch.  See include/gdn.h.
#include <stdint.h>

#include "gdn_internal.cuh"

namespace {

thread_local int g_last_cuda_error = 0;
constexpr int kMaxDecodeTokens = 64;   // gdn_decode_tokens: tokens per call
constexpr int kMaxSegments = 16;       // gdn_chunk_fwd_split: segments per sequence
// Prefill kernel choice of the calling thread (a per-thread setting: one thread's
// choice never changes what another thread's calls run).
thread_local int g_prefill_kernel = GDN_PREFILL_AUTO;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

gdn_status cuda_status(cudaError_t err)
{
    if (err == cudaSuccess) return GDN_OK;
    g_last_cuda_error = (int)err;
    return GDN_ERR_CUDA;
}

// Shape checks common to both entry points.
gdn_status check_heads(int Hqk, int Hv, int dk, int dv)
{
    if (Hqk <= 0 || Hv <= 0 || dk <= 0 || dv <= 0) return GDN_ERR_INVALID_ARG;
    if (Hv % Hqk != 0) return GDN_ERR_UNSUPPORTED;
    if (dk != gdn::kHeadDim || dv != gdn::kHeadDim) return GDN_ERR_UNSUPPORTED;
    return GDN_OK;
}

// The prefill kernel a call with these sizes runs under the current choice, or
// -1 when a forced tensor-core kernel cannot take the call.
int resolve_prefill_kernel(int B, int Hv, gdn_dtype dtype)
{
    (void)B;
    (void)Hv;
    const int kind = g_prefill_kernel;
    const bool tc_ok = dtype == GDN_BF16 && gdn::chunk_tc_available();
    if (kind == GDN_PREFILL_AUTO) return tc_ok ? GDN_PREFILL_TC : GDN_PREFILL_SIMT;
    if (kind != GDN_PREFILL_SIMT && !tc_ok) return -1;
    return kind;
}

// Shared by the two prefill entry points: B sequences of T tokens each, or, with
// cu_seqlens, B packed sequences in T token rows.
gdn_status chunk_fwd_common(const void *q, const void *k, const void *v,
                            const float *alpha, const float *beta, const float *S0,
                            void *o, float *S_final, const int *cu_seqlens,
                            int B, int T, int Hqk, int Hv, int dk, int dv, int chunk,
                            gdn_dtype dtype, void *stream)
{
    if (B < 0 || T < 0) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    gdn_status st = check_heads(Hqk, Hv, dk, dv);
    if (st != GDN_OK) return st;
    if (chunk != gdn::kChunk) return GDN_ERR_UNSUPPORTED;
    if (B > 65535) return GDN_ERR_UNSUPPORTED;
    if (B == 0) return GDN_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t state_bytes = (size_t)B * Hv * dk * dv * sizeof(float);
    if (T == 0) {   // every sequence is empty: the state passes through
        if (!S_final) return GDN_OK;
        if (!aligned16(S_final) || (S0 && !aligned16(S0))) return GDN_ERR_INVALID_ARG;
        if (S0 == S_final) return GDN_OK;
        return cuda_status(S0 ? cudaMemcpyAsync(S_final, S0, state_bytes, cudaMemcpyDeviceToDevice, s)
                              : cudaMemsetAsync(S_final, 0, state_bytes, s));
    }
    if (!q || !k || !v || !alpha || !beta || !o) return GDN_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, alpha, beta, S0, o, S_final};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_INVALID_ARG;

    gdn::ChunkArgs a{q, k, v, alpha, beta, S0, o, S_final, B, T, Hqk, Hv};
    a.cu_seqlens = cu_seqlens;
    const int kind = resolve_prefill_kernel(B, Hv, dtype);
    if (kind < 0) return GDN_ERR_UNSUPPORTED;
    cudaError_t err;
    switch (kind) {
    case GDN_PREFILL_TC: err = gdn::launch_chunk_tc(a, s); break;
    default: err = gdn::launch_chunk_simt(a, dtype, s); break;
    }
    return cuda_status(err);
}

}  // namespace

extern "C" {

gdn_status gdn_chunk_fwd(const void *q, const void *k, const void *v,
                         const float *alpha, const float *beta, const float *S0,
                         void *o, float *S_final,
                         int B, int T, int Hqk, int Hv, int dk, int dv, int chunk,
                         gdn_dtype dtype, void *stream)
{
    return chunk_fwd_common(q, k, v, alpha, beta, S0, o, S_final, nullptr, B, T, Hqk, Hv, dk, dv,
                            chunk, dtype, stream);
}

gdn_status gdn_chunk_fwd_varlen(const void *q, const void *k, const void *v,
                                const float *alpha, const float *beta, const float *S0,
                                void *o, float *S_final, const int *cu_seqlens,
                                int N, int T_total, int Hqk, int Hv, int dk, int dv, int chunk,
                                gdn_dtype dtype, void *stream)
{
    if (N > 0 && T_total > 0 && (!cu_seqlens || (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)))
        return GDN_ERR_INVALID_ARG;
    return chunk_fwd_common(q, k, v, alpha, beta, S0, o, S_final, cu_seqlens, N, T_total, Hqk, Hv,
                            dk, dv, chunk, dtype, stream);
}

gdn_status gdn_decode_step(const void *q, const void *k, const void *v,
                           const float *alpha, const float *beta, const float *S,
                           void *o, float *S_new,
                           int B, int Hqk, int Hv, int dk, int dv,
                           gdn_dtype dtype, void *stream)
{
    if (B < 0) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    gdn_status st = check_heads(Hqk, Hv, dk, dv);
    if (st != GDN_OK) return st;
    if (B == 0) return GDN_OK;
    if ((long long)B * Hv > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
    if (!q || !k || !v || !alpha || !beta || !S || !o || !S_new) return GDN_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, alpha, beta, S, o, S_new};
    for (const void *p : ptrs)
        if (!aligned16(p)) return GDN_ERR_INVALID_ARG;
    gdn::DecodeArgs a{q, k, v, alpha, beta, S, o, S_new, B, Hqk, Hv};
    return cuda_status(gdn::launch_decode(a, dtype, static_cast<cudaStream_t>(stream)));
}

gdn_status gdn_set_prefill_kernel(gdn_prefill_kernel kernel)
{
    const int k = (int)kernel;
    if (k < GDN_PREFILL_AUTO || k > GDN_PREFILL_TC) return GDN_ERR_INVALID_ARG;
    g_prefill_kernel = k;
    return GDN_OK;
}

gdn_prefill_kernel gdn_get_prefill_kernel(void)
{
    return (gdn_prefill_kernel)g_prefill_kernel;
}

int gdn_prefill_kernel_for(int B, int Hv, gdn_dtype dtype)
{
    if (B < 0 || Hv <= 0 || (dtype != GDN_F32 && dtype != GDN_BF16)) return -1;
    return resolve_prefill_kernel(B, Hv, dtype);
}

gdn_status gdn_decode_tokens(const void *q, const void *k, const void *v,
                             const float *alpha, const float *beta, const float *S,
                             void *o, float *S_new, float *S_steps,
                             int B, int n, int Hqk, int Hv, int dk, int dv,
                             gdn_dtype dtype, void *stream)
{
    if (B < 0 || n < 1) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    gdn_status st = check_heads(Hqk, Hv, dk, dv);
    if (st != GDN_OK) return st;
    if (n > kMaxDecodeTokens) return GDN_ERR_UNSUPPORTED;
    if (B == 0) return GDN_OK;
    if ((long long)B * Hv > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
    if (!q || !k || !v || !alpha || !beta || !S || !o || !S_new) return GDN_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, alpha, beta, S, o, S_new, S_steps};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_INVALID_ARG;
    gdn::DecodeArgs a{q, k, v, alpha, beta, S, o, S_new, B, Hqk, Hv};
    a.ntok = n;
    a.S_steps = S_steps;
    return cuda_status(gdn::launch_decode(a, dtype, static_cast<cudaStream_t>(stream)));
}

gdn_status gdn_decode_step_slots(const void *q, const void *k, const void *v,
                                 const float *alpha, const float *beta,
                                 float *state_pool, const int *slots, void *o,
                                 int B, int n_slots, int Hqk, int Hv, int dk, int dv,
                                 gdn_dtype dtype, void *stream)
{
    if (B < 0 || n_slots < 0) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    gdn_status st = check_heads(Hqk, Hv, dk, dv);
    if (st != GDN_OK) return st;
    if (B == 0) return GDN_OK;
    if ((long long)B * Hv > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
    if (!q || !k || !v || !alpha || !beta || !slots || !o || (n_slots > 0 && !state_pool))
        return GDN_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, alpha, beta, state_pool, o};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(slots) & 3u) return GDN_ERR_INVALID_ARG;
    gdn::DecodeArgs a{q, k, v, alpha, beta, state_pool, o, state_pool, B, Hqk, Hv};
    a.slots = slots;
    a.n_slots = n_slots;
    return cuda_status(gdn::launch_decode(a, dtype, static_cast<cudaStream_t>(stream)));
}

namespace {

// Most segments whose CTAs (B*Hv*(2S-1): first runs plus transition runs) all fit
// on the device at once; 1 when even two do not.
int auto_segments(int B, int Hv)
{
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return 1;
    }
    int S = 1;
    while (S < kMaxSegments && (long long)B * Hv * (2 * (S + 1) - 1) <= sms) ++S;
    return S;
}

}  // namespace

}  // extern "C"

namespace gdn {

// Scratch bytes gdn_chunk_fwd_split will use for these arguments under the calling
// thread's kernel choice: 0 when the call goes straight to gdn_chunk_fwd (not bf16,
// the tensor cores unavailable or not chosen, or one segment covers the sequence).
size_t split_scratch_needed(int B, int T, int Hv, int dk, int dv, int segments, gdn_dtype dtype)
{
    if (segments < 0 || segments > kMaxSegments) return 0;
    if (segments == 0 && B > 0 && Hv > 0) segments = auto_segments(B, Hv);
    const bool tc = dtype == GDN_BF16 && chunk_tc_available() && g_prefill_kernel != GDN_PREFILL_SIMT;
    if (!tc || B <= 0 || T <= 0 || Hv <= 0 || segments <= 1 || dk != kHeadDim || dv != kHeadDim) return 0;
    return chunk_tc_split_workspace(B, T, Hv, segments);
}

}  // namespace gdn

extern "C" {

size_t gdn_chunk_fwd_split_workspace(int B, int T, int Hv, int dk, int dv, int segments)
{
    if (B <= 0 || T <= 0 || Hv <= 0 || dk != gdn::kHeadDim || dv != gdn::kHeadDim) return 0;
    if (segments == 0) segments = auto_segments(B, Hv);
    if (segments < 1 || segments > kMaxSegments) return 0;
    return gdn::chunk_tc_split_workspace(B, T, Hv, segments);
}

gdn_status gdn_chunk_fwd_split(const void *q, const void *k, const void *v,
                               const float *alpha, const float *beta, const float *S0,
                               void *o, float *S_final,
                               int B, int T, int Hqk, int Hv, int dk, int dv, int chunk,
                               int segments, gdn_dtype dtype, void *workspace,
                               size_t workspace_bytes, void *stream)
{
    if (segments < 0 || segments > kMaxSegments) return GDN_ERR_INVALID_ARG;
    if (segments == 0 && B > 0 && Hv > 0) segments = auto_segments(B, Hv);
    const size_t need = gdn::split_scratch_needed(B, T, Hv, dk, dv, segments, dtype);
    if (need == 0)   // nothing to split
        return gdn_chunk_fwd(q, k, v, alpha, beta, S0, o, S_final, B, T, Hqk, Hv, dk, dv, chunk,
                             dtype, stream);
    if (B < 0 || T < 0) return GDN_ERR_INVALID_ARG;
    gdn_status st = check_heads(Hqk, Hv, dk, dv);
    if (st != GDN_OK) return st;
    if (chunk != gdn::kChunk) return GDN_ERR_UNSUPPORTED;
    if ((long long)B * (2 * segments - 1) > 65535) return GDN_ERR_UNSUPPORTED;
    if (!q || !k || !v || !alpha || !beta || !o) return GDN_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, alpha, beta, S0, o, S_final};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return GDN_ERR_INVALID_ARG;
    gdn::ChunkArgs a{q, k, v, alpha, beta, S0, o, S_final, B, T, Hqk, Hv};
    return cuda_status(gdn::launch_chunk_tc_split(a, segments, workspace,
                                                  static_cast<cudaStream_t>(stream)));
}

size_t gdn_chunk_fwd_pipelined_workspace(int B, int Hqk, int Hv, int dk, int dv)
{
    if (dk != gdn::kHeadDim || dv != gdn::kHeadDim) return 0;
    return gdn::chunk_pipe_workspace(B, Hqk, Hv);
}

gdn_status gdn_chunk_fwd_pipelined(const void *q, const void *k, const void *v,
                                   const float *alpha, const float *beta, const float *S0,
                                   void *o, float *S_final,
                                   int B, int T, int Hqk, int Hv, int dk, int dv, int chunk,
                                   gdn_dtype dtype, const gdn_pipeline_options *opts,
                                   void *workspace, size_t workspace_bytes, void *stream)
{
    if (opts && (opts->chain_ctas < 0 || opts->wait_limit_cycles < 0)) return GDN_ERR_INVALID_ARG;
    // fp32 inputs, empty problems and builds without the tensor-map encoder take the
    // plain prefill (same function; the workspace is not used)
    if (dtype != GDN_BF16 || B <= 0 || T <= 0 || !gdn::chunk_tc_available())
        return gdn_chunk_fwd(q, k, v, alpha, beta, S0, o, S_final, B, T, Hqk, Hv, dk, dv, chunk,
                             dtype, stream);
    gdn_status st = check_heads(Hqk, Hv, dk, dv);
    if (st != GDN_OK) return st;
    if (chunk != gdn::kChunk) return GDN_ERR_UNSUPPORTED;
    if (B > 65535) return GDN_ERR_UNSUPPORTED;
    if (!q || !k || !v || !alpha || !beta || !o) return GDN_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, alpha, beta, S0, o, S_final};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_INVALID_ARG;
    const size_t need = gdn::chunk_pipe_workspace(B, Hqk, Hv);
    if (need == 0) return GDN_ERR_UNSUPPORTED;
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return GDN_ERR_INVALID_ARG;
    gdn::ChunkArgs a{q, k, v, alpha, beta, S0, o, S_final, B, T, Hqk, Hv};
    return cuda_status(gdn::launch_chunk_pipe(a, opts ? opts->chain_ctas : 0,
                                              opts ? opts->wait_limit_cycles : 0, workspace,
                                              workspace_bytes, static_cast<cudaStream_t>(stream)));
}

gdn_status gdn_device_status(void *stream)
{
    cudaError_t err = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (err != cudaSuccess) return cuda_status(err);
    unsigned a = 0, b = 0, c = 0;
    err = gdn::chunk_pipe_take_error(&a);
    if (err == cudaSuccess) err = gdn::chunk_tc_take_error(&b);
    if (err == cudaSuccess) err = gdn::split_take_error(&c);
    if (err != cudaSuccess) return cuda_status(err);
    return (a | b | c) ? GDN_ERR_TIMEOUT : GDN_OK;
}

const char *gdn_status_string(gdn_status status)
{
    switch (status) {
    case GDN_OK: return "GDN_OK";
    case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG";
    case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED";
    case GDN_ERR_CUDA: return "GDN_ERR_CUDA";
    case GDN_ERR_TIMEOUT: return "GDN_ERR_TIMEOUT";
    }
    return "GDN_UNKNOWN_STATUS";
}

int gdn_last_cuda_error(void) { return g_last_cuda_error; }

int gdn_version(void) { return 200; }

}  // extern "C"

extern "C" {

size_t gdn_bwd_workspace(int B, int T, int Hv, int dk, int dv)
{
    if (dk != gdn::kHeadDim || dv != gdn::kHeadDim) return 0;
    return gdn::bwd_workspace(B, T, Hv);
}

gdn_status gdn_bwd(const void *q, const void *k, const void *v, const float *alpha,
                   const float *beta, const float *S0, const void *dO, const float *dS_final,
                   float *dq, float *dk, float *dv, float *dalpha, float *dbeta, float *dS0,
                   int B, int T, int Hqk, int Hv, int dk_, int dv_, gdn_dtype dtype,
                   void *workspace, size_t workspace_bytes, void *stream)
{
    if (B < 0 || T < 0) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    gdn_status st = check_heads(Hqk, Hv, dk_, dv_);
    if (st != GDN_OK) return st;
    if (B == 0) return GDN_OK;
    if (B > 65535 || (long long)Hv * 4 > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
    if (!dS0) return GDN_ERR_INVALID_ARG;
    if (T > 0 && (!q || !k || !v || !alpha || !beta || !dO || !dq || !dk || !dv || !dalpha || !dbeta))
        return GDN_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, alpha, beta, S0, dO, dS_final, dq, dk, dv, dalpha, dbeta, dS0};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_INVALID_ARG;
    const size_t need = gdn::bwd_workspace(B, T, Hv);
    if (need > 0 && (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u)))
        return GDN_ERR_INVALID_ARG;
    gdn::BwdLaunch L{q, k, v, dO, alpha, beta, S0, dS_final, dq, dk, dv, dalpha, dbeta, dS0,
                     static_cast<float *>(workspace), B, T, Hqk, Hv};
    return cuda_status(gdn::launch_bwd(L, dtype, static_cast<cudaStream_t>(stream)));
}

size_t gdn_bwd_chunk_workspace(int B, int T, int Hv, int dk, int dv)
{
    if (dk != gdn::kHeadDim || dv != gdn::kHeadDim) return 0;
    return gdn::bwd_chunk_workspace(B, T, Hv);
}

gdn_status gdn_bwd_chunk(const void *q, const void *k, const void *v, const float *alpha,
                         const float *beta, const float *S0, const void *dO, const float *dS_final,
                         float *dq, float *dk, float *dv, float *dalpha, float *dbeta, float *dS0,
                         int B, int T, int Hqk, int Hv, int dk_, int dv_, gdn_dtype dtype,
                         void *workspace, size_t workspace_bytes, void *stream)
{
    if (B < 0 || T < 0) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    gdn_status st = check_heads(Hqk, Hv, dk_, dv_);
    if (st != GDN_OK) return st;
    if (dtype != GDN_BF16) return GDN_ERR_UNSUPPORTED;
    if (B == 0) return GDN_OK;
    if (B > 65535 || Hqk > 65535 || Hv > 65535) return GDN_ERR_UNSUPPORTED;
    if (!dS0) return GDN_ERR_INVALID_ARG;
    if (T > 0 && (!q || !k || !v || !alpha || !beta || !dO || !dq || !dk || !dv || !dalpha || !dbeta))
        return GDN_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, alpha, beta, S0, dO, dS_final, dq, dk, dv, dalpha, dbeta, dS0};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_INVALID_ARG;
    const size_t need = gdn::bwd_chunk_workspace(B, T, Hv);
    if (need > 0 && (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u)))
        return GDN_ERR_INVALID_ARG;
    gdn::BwdLaunch L{q, k, v, dO, alpha, beta, S0, dS_final, dq, dk, dv, dalpha, dbeta, dS0,
                     static_cast<float *>(workspace), B, T, Hqk, Hv};
    return cuda_status(gdn::launch_bwd_chunk(L, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
