// Decode: one token of the gated delta rule for every (sequence, V head).
//
// Source: "Qwen3.8-Flash-Next 技术总结 -- Qwen4 架构的探路者", section 2.1 "Gated
// DeltaNet", first form of the update.  For one token and one head, with S the
// 128 x 128 fp32 state (row = key dim):
//   p = S^T k,  r = S^T q,  s = k . q
//   u = beta (v - alpha p)
//   S' = alpha S + k u^T
//   o  = S'^T q = alpha r + s u
// The state is the whole cost: it is read once and written once (in place), so
// the kernel is an HBM stream.  The same kernel runs n tokens per sequence
// (multi-token decode / draft verification), the state staying in registers
// between tokens, and can gather states from a pool by slot index.
// One CTA of 256 threads owns one (b, h) state
// (64 KiB): warp w holds rows w, w+8, ..., w+120 and lane l holds columns
// 4l..4l+3, i.e. 16 float4 per thread kept in registers between the load and the
// store.  Every warp-wide access is one contiguous 512-byte row.  Column sums
// over the 8 warps go through shared memory.
#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int kDecodeThreads = 256;
constexpr int kRowsPerThread = kHeadDim / (kDecodeThreads / 32);  // 16

__device__ __forceinline__ float4 ld_stream(const float4 *p) { return __ldcs(p); }
__device__ __forceinline__ void st_stream(float4 *p, float4 v) { __stcs(p, v); }

// n tokens per (b, h) in sequence, the state held in registers throughout; the
// token inputs are [B, n, H, 128] (gates [B, n, Hv]).  Optional: S_steps gets
// the state after every token ([B, n, Hv, 128, 128]); slots maps sequence b to
// its state in a pool of n_slots states (a slot outside [0, n_slots) skips b).
// kMulti = false is the one-token form (ntok == 1, S_steps null): the state update
// and its store are one loop, as the HBM stream wants.
template <typename T, bool kMulti>
__global__ void __launch_bounds__(kDecodeThreads, 2)
decode_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
              const float *__restrict__ alpha, const float *__restrict__ beta,
              const float *S, T *__restrict__ o, float *S_new, float *__restrict__ S_steps,
              const int *__restrict__ slots, int n_slots, int ntok, int Hqk, int Hv)
{
    const int bh = blockIdx.x;                  // b * Hv + h
    const int b = bh / Hv, h = bh - b * Hv;
    const int hq = h / (Hv / Hqk);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    __shared__ float sk[kHeadDim], sq[kHeadDim];
    __shared__ float4 sp[8][32], sr[8][32];
    __shared__ float skq;

    size_t state = (size_t)bh;                  // index of the (b, h) state
    if (slots) {
        const int sl = slots[b];
        if (sl < 0 || sl >= n_slots) return;    // padding entry: nothing to do
        state = (size_t)sl * Hv + h;
    }
    // Issue the state loads first: they are the latency that matters.
    const size_t base = state * kHeadDim * kHeadDim;
    const float4 *S4 = reinterpret_cast<const float4 *>(S + base);
    float4 s[kRowsPerThread];
#pragma unroll
    for (int m = 0; m < kRowsPerThread; ++m) s[m] = ld_stream(S4 + (warp + 8 * m) * 32 + lane);

    if (!kMulti) ntok = 1;
    float4 *D4 = reinterpret_cast<float4 *>(S_new + base);
#pragma unroll 1
    for (int t = 0; t < ntok; ++t) {
        const size_t tok = (size_t)b * ntok + t;            // token row in [B, n, ...]
        const size_t qk_off = (tok * Hqk + hq) * kHeadDim;
        const size_t gi = tok * Hv + h;
        if (t > 0) __syncthreads();                          // sk, sq, sp, sr reused
        if (tid < kHeadDim) sk[tid] = to_f32(k[qk_off + tid]);
        else sq[tid - kHeadDim] = to_f32(q[qk_off + tid - kHeadDim]);
        const float a = alpha[gi], be = beta[gi];
        __syncthreads();

        if (warp == 0) {  // s = k . q
            float acc = 0.f;
#pragma unroll
            for (int i = lane; i < kHeadDim; i += 32) acc = fmaf(sk[i], sq[i], acc);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            if (lane == 0) skq = acc;
        }
        float4 pp = make_float4(0.f, 0.f, 0.f, 0.f), rr = pp;
#pragma unroll
        for (int m = 0; m < kRowsPerThread; ++m) {
            const float ki = sk[warp + 8 * m], qi = sq[warp + 8 * m];
            pp.x = fmaf(s[m].x, ki, pp.x); pp.y = fmaf(s[m].y, ki, pp.y);
            pp.z = fmaf(s[m].z, ki, pp.z); pp.w = fmaf(s[m].w, ki, pp.w);
            rr.x = fmaf(s[m].x, qi, rr.x); rr.y = fmaf(s[m].y, qi, rr.y);
            rr.z = fmaf(s[m].z, qi, rr.z); rr.w = fmaf(s[m].w, qi, rr.w);
        }
        sp[warp][lane] = pp;
        sr[warp][lane] = rr;
        __syncthreads();

        float4 p = sp[0][lane], r = sr[0][lane];
#pragma unroll
        for (int w = 1; w < 8; ++w) {
            const float4 pw = sp[w][lane], rw = sr[w][lane];
            p.x += pw.x; p.y += pw.y; p.z += pw.z; p.w += pw.w;
            r.x += rw.x; r.y += rw.y; r.z += rw.z; r.w += rw.w;
        }
        const size_t v_off = gi * kHeadDim + 4 * lane;
        float4 u;
        u.x = be * (to_f32(v[v_off + 0]) - a * p.x);
        u.y = be * (to_f32(v[v_off + 1]) - a * p.y);
        u.z = be * (to_f32(v[v_off + 2]) - a * p.z);
        u.w = be * (to_f32(v[v_off + 3]) - a * p.w);
        if (warp == 0) {
            const float kq = skq;
            o[v_off + 0] = from_f32<T>(fmaf(kq, u.x, a * r.x));
            o[v_off + 1] = from_f32<T>(fmaf(kq, u.y, a * r.y));
            o[v_off + 2] = from_f32<T>(fmaf(kq, u.z, a * r.z));
            o[v_off + 3] = from_f32<T>(fmaf(kq, u.w, a * r.w));
        }
        float4 *P4 = (kMulti && S_steps) ? reinterpret_cast<float4 *>(S_steps + gi * kHeadDim * kHeadDim)
                                         : nullptr;
#pragma unroll
        for (int m = 0; m < kRowsPerThread; ++m) {
            const float ki = sk[warp + 8 * m];
            s[m].x = fmaf(a, s[m].x, ki * u.x);
            s[m].y = fmaf(a, s[m].y, ki * u.y);
            s[m].z = fmaf(a, s[m].z, ki * u.z);
            s[m].w = fmaf(a, s[m].w, ki * u.w);
            if (!kMulti) st_stream(D4 + (warp + 8 * m) * 32 + lane, s[m]);
            else if (P4) st_stream(P4 + (warp + 8 * m) * 32 + lane, s[m]);
        }
    }
    if (kMulti) {
#pragma unroll
        for (int m = 0; m < kRowsPerThread; ++m) st_stream(D4 + (warp + 8 * m) * 32 + lane, s[m]);
    }
}

template <typename T, bool kMulti>
void launch_typed(const DecodeArgs &a, cudaStream_t stream)
{
    const unsigned grid = (unsigned)((size_t)a.B * a.Hv);
    decode_kernel<T, kMulti><<<grid, kDecodeThreads, 0, stream>>>(
        (const T *)a.q, (const T *)a.k, (const T *)a.v, a.alpha, a.beta, a.S, (T *)a.o, a.S_new,
        a.S_steps, a.slots, a.n_slots, a.ntok, a.Hqk, a.Hv);
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs &a, gdn_dtype dtype, cudaStream_t stream)
{
    const bool multi = a.ntok != 1 || a.S_steps;
    if (dtype == GDN_BF16) {
        if (multi) launch_typed<__nv_bfloat16, true>(a, stream);
        else launch_typed<__nv_bfloat16, false>(a, stream);
    } else {
        if (multi) launch_typed<float, true>(a, stream);
        else launch_typed<float, false>(a, stream);
    }
    return cudaGetLastError();
}

}  // namespace gdn
