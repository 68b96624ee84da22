// Chunkwise (WY) prefill on CUDA cores, fp32 arithmetic.  This is the fp32 path
// of gdn_chunk_fwd (inputs in fp32 must match the recurrence to 1e-4 relative,
// which tensor-core bf16/tf32 products cannot).
//
// Source: "Qwen3.8-Flash-Next 技术总结 -- Qwen4 架构的探路者", section 2.1 "Gated
// DeltaNet": the update S_t = alpha_t S_{t-1} + beta_t k_t (v_t - alpha_t S_{t-1}^T k_t)^T
// evaluated chunk by chunk with the WY representation (the page names the method;
// the blocked equations are derived from the update).  For a chunk of C = 64
// tokens starting from state S (dk x dv), with b_r = sum_{j<=r} log alpha_j,
// gamma_r = exp(b_r) and Gam[r,i] = exp(b_r - b_i) (i <= r):
//   A[r,i]  = beta_r Gam[r,i] (k_r . k_i)                 i < r
//   (I + A) [W | U~] = [diag(beta gamma) K | diag(beta) V]  (forward substitution)
//   U       = U~ - W S
//   O       = diag(gamma) Q S + (Gam o Q K^T) U            (i <= r)
//   S      <- gamma_{C-1} S + K~^T U,   K~_i = exp(b_{C-1} - b_i) k_i
// A partial last chunk is padded with k = q = v = 0, alpha = 1, beta = 0, which
// leaves every quantity of the real tokens unchanged.
//
// Grid: one CTA per (b, V head, dv slice of 64 columns); the columns of S evolve
// independently (the update mixes only key rows), so the slices need no
// communication.  Everything of a chunk lives in shared memory.
#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int C = kChunk;          // 64
constexpr int D = kHeadDim;        // 128 (dk)
constexpr int DVS = 64;            // dv columns per CTA
constexpr int NT = 256;            // threads per CTA
constexpr int PAD = 68;            // row stride (floats) of the 64-wide tiles

struct Smem {
    float Kt[D][PAD];      // K^T: [d][r]
    float Qt[D][PAD];      // Q^T: [d][r]
    float Wt[D][PAD];      // W^T: [d][r]
    float S[D][PAD];       // state slice: [d][j], j < DVS
    float U[C][PAD];       // V -> U~ -> U: [r][j]
    float Pt[C][PAD];      // (Gam o Q K^T)^T masked to i <= r: [i][r]
    float A[C][C];         // strictly lower A: [r][i]
    float bcum[C], gamma[C], beta[C], gtail[C];
};

template <typename T>
__global__ void __launch_bounds__(NT, 1)
chunk_simt_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                  const float *__restrict__ alpha, const float *__restrict__ beta,
                  const float *S0, T *__restrict__ o, float *S_final, int Tlen, int Hqk, int Hv,
                  const int *__restrict__ cu_seqlens)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw);

    const int nslice = kHeadDim / DVS;
    const int h = blockIdx.x / nslice, slice = blockIdx.x % nslice;
    const int b = blockIdx.y;
    const int hq = h / (Hv / Hqk);
    const int j_base = slice * DVS;
    const int tid = threadIdx.x;
    // token rows of this sequence: [bt * Tlen + tb, ... + Lseq) of the token arrays
    int tb = 0, Lseq = Tlen, bt = b;
    if (cu_seqlens) {   // packed sequences; offsets clamped into [0, Tlen]
        const int s0 = min(max(cu_seqlens[b], 0), Tlen);
        tb = s0;
        Lseq = min(max(cu_seqlens[b + 1], s0), Tlen) - s0;
        bt = 0;
    }

    // ---- initial state slice
    const size_t s_off = ((size_t)b * Hv + h) * D * kHeadDim;
    for (int e = tid; e < D * DVS; e += NT) {
        const int d = e / DVS, j = e % DVS;
        sm.S[d][j] = S0 ? S0[s_off + (size_t)d * kHeadDim + j_base + j] : 0.f;
    }

    // thread tiles
    const int r0 = (tid / 16) * 4;     // 4 rows of a 64 x 64 tile
    const int c0 = (tid % 16) * 4;     // 4 columns
    const int d0 = (tid / 16) * 8;     // 8 state rows of the 128 x 64 state update

    for (int t0 = 0; t0 < Lseq; t0 += C) {
        const int L = min(C, Lseq - t0);
        __syncthreads();  // previous chunk fully consumed

        // ---- load the chunk (transposed K, Q; V slice), padding rows >= L
        for (int e = tid; e < C * D; e += NT) {
            const int r = e / D, d = e % D;
            float kv = 0.f, qv = 0.f;
            if (r < L) {
                const size_t off = (((size_t)bt * Tlen + tb + t0 + r) * Hqk + hq) * D + d;
                kv = to_f32(k[off]);
                qv = to_f32(q[off]);
            }
            sm.Kt[d][r] = kv;
            sm.Qt[d][r] = qv;
        }
        for (int e = tid; e < C * DVS; e += NT) {
            const int r = e / DVS, j = e % DVS;
            sm.U[r][j] = r < L ? to_f32(v[(((size_t)bt * Tlen + tb + t0 + r) * Hv + h) * kHeadDim + j_base + j]) : 0.f;
        }
        if (tid < 32) {  // gates and the chunk-local cumulative log decay (warp scan)
            const int lane = tid;
            float la[2], be[2];
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                const int r = 2 * lane + x;
                const size_t g = ((size_t)bt * Tlen + tb + t0 + r) * Hv + h;
                la[x] = r < L ? clamped_log(alpha[g]) : 0.f;
                be[x] = r < L ? beta[g] : 0.f;
            }
            float incl = la[0] + la[1];
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += y;
            }
            const float excl = incl - (la[0] + la[1]);
            const float bc0 = excl + la[0], bc1 = incl;
            const float blast = __shfl_sync(0xffffffffu, incl, 31);
            sm.bcum[2 * lane] = bc0;
            sm.bcum[2 * lane + 1] = bc1;
            sm.gamma[2 * lane] = expf(bc0);
            sm.gamma[2 * lane + 1] = expf(bc1);
            sm.beta[2 * lane] = be[0];
            sm.beta[2 * lane + 1] = be[1];
            sm.gtail[2 * lane] = expf(blast - bc0);
            sm.gtail[2 * lane + 1] = expf(blast - bc1);
        }
        __syncthreads();

        // ---- grams K K^T and Q K^T on the 4 x 4 tile (r0.., c0.. as i), then A and P
        {
            float gk[4][4] = {}, gq[4][4] = {};
            for (int d = 0; d < D; ++d) {
                const float4 kr = *reinterpret_cast<const float4 *>(&sm.Kt[d][r0]);
                const float4 qr = *reinterpret_cast<const float4 *>(&sm.Qt[d][r0]);
                const float4 ki = *reinterpret_cast<const float4 *>(&sm.Kt[d][c0]);
                const float a_k[4] = {kr.x, kr.y, kr.z, kr.w};
                const float a_q[4] = {qr.x, qr.y, qr.z, qr.w};
                const float bb[4] = {ki.x, ki.y, ki.z, ki.w};
#pragma unroll
                for (int x = 0; x < 4; ++x)
#pragma unroll
                    for (int y = 0; y < 4; ++y) {
                        gk[x][y] = fmaf(a_k[x], bb[y], gk[x][y]);
                        gq[x][y] = fmaf(a_q[x], bb[y], gq[x][y]);
                    }
            }
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) {
                    const int r = r0 + x, i = c0 + y;
                    // mask before exp: b_r - b_i is only formed for i <= r
                    const float dec = i <= r ? expf(sm.bcum[r] - sm.bcum[i]) : 0.f;
                    sm.A[r][i] = i < r ? sm.beta[r] * dec * gk[x][y] : 0.f;
                    sm.Pt[i][r] = dec * gq[x][y];
                }
        }
        __syncthreads();

        // ---- forward substitution, one right-hand-side column per thread:
        //      threads 0..127 -> column d of W, threads 128..191 -> column j of U~
        if (tid < D + DVS) {
            float x[C];
            if (tid < D) {
#pragma unroll
                for (int r = 0; r < C; ++r) x[r] = sm.beta[r] * sm.gamma[r] * sm.Kt[tid][r];
            } else {
#pragma unroll
                for (int r = 0; r < C; ++r) x[r] = sm.beta[r] * sm.U[r][tid - D];
            }
#pragma unroll
            for (int r = 1; r < C; ++r) {
                float acc = x[r];
#pragma unroll
                for (int i = 0; i < r; ++i) acc = fmaf(-sm.A[r][i], x[i], acc);
                x[r] = acc;
            }
            if (tid < D) {
#pragma unroll
                for (int r = 0; r < C; ++r) sm.Wt[tid][r] = x[r];
            } else {
#pragma unroll
                for (int r = 0; r < C; ++r) sm.U[r][tid - D] = x[r];
            }
        }
        __syncthreads();

        // ---- U = U~ - W S and QS = Q S on the 4 x 4 tile (rows r0.., columns c0..)
        float qs[4][4] = {};
        {
            float ws[4][4] = {};
            for (int d = 0; d < D; ++d) {
                const float4 w = *reinterpret_cast<const float4 *>(&sm.Wt[d][r0]);
                const float4 qq = *reinterpret_cast<const float4 *>(&sm.Qt[d][r0]);
                const float4 s4 = *reinterpret_cast<const float4 *>(&sm.S[d][c0]);
                const float aw[4] = {w.x, w.y, w.z, w.w};
                const float aq[4] = {qq.x, qq.y, qq.z, qq.w};
                const float bs[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
                for (int x = 0; x < 4; ++x)
#pragma unroll
                    for (int y = 0; y < 4; ++y) {
                        ws[x][y] = fmaf(aw[x], bs[y], ws[x][y]);
                        qs[x][y] = fmaf(aq[x], bs[y], qs[x][y]);
                    }
            }
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) sm.U[r0 + x][c0 + y] -= ws[x][y];
        }
        __syncthreads();

        // ---- O = diag(gamma) Q S + P U  (P[r,i] = Pt[i][r], zero for i > r)
        {
            float acc[4][4];
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) acc[x][y] = sm.gamma[r0 + x] * qs[x][y];
            const int imax = min(r0 + 4, C);
            for (int i = 0; i < imax; ++i) {
                const float4 p = *reinterpret_cast<const float4 *>(&sm.Pt[i][r0]);
                const float4 u = *reinterpret_cast<const float4 *>(&sm.U[i][c0]);
                const float ap[4] = {p.x, p.y, p.z, p.w};
                const float bu[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int x = 0; x < 4; ++x)
#pragma unroll
                    for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(ap[x], bu[y], acc[x][y]);
            }
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const int r = r0 + x;
                if (r < L) {
                    T *dst = o + (((size_t)bt * Tlen + tb + t0 + r) * Hv + h) * kHeadDim + j_base + c0;
#pragma unroll
                    for (int y = 0; y < 4; ++y) dst[y] = from_f32<T>(acc[x][y]);
                }
            }
        }
        // ---- S <- gamma_{C-1} S + K~^T U on the 8 x 4 tile (state rows d0.., columns c0..)
        {
            const float glast = sm.gamma[C - 1];
            float acc[8][4];
#pragma unroll
            for (int x = 0; x < 8; ++x) {
                const float4 s4 = *reinterpret_cast<const float4 *>(&sm.S[d0 + x][c0]);
                acc[x][0] = glast * s4.x; acc[x][1] = glast * s4.y;
                acc[x][2] = glast * s4.z; acc[x][3] = glast * s4.w;
            }
            for (int i = 0; i < C; ++i) {
                const float gi = sm.gtail[i];
                const float4 u = *reinterpret_cast<const float4 *>(&sm.U[i][c0]);
                const float bu[4] = {gi * u.x, gi * u.y, gi * u.z, gi * u.w};
#pragma unroll
                for (int x = 0; x < 8; ++x) {
                    const float kd = sm.Kt[d0 + x][i];
#pragma unroll
                    for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(kd, bu[y], acc[x][y]);
                }
            }
#pragma unroll
            for (int x = 0; x < 8; ++x)
                *reinterpret_cast<float4 *>(&sm.S[d0 + x][c0]) =
                    make_float4(acc[x][0], acc[x][1], acc[x][2], acc[x][3]);
        }
    }
    __syncthreads();
    if (S_final) {
        for (int e = tid; e < D * DVS; e += NT) {
            const int d = e / DVS, j = e % DVS;
            S_final[s_off + (size_t)d * kHeadDim + j_base + j] = sm.S[d][j];
        }
    }
}

template <typename T>
cudaError_t launch_typed(const ChunkArgs &a, cudaStream_t stream)
{
    const size_t smem = sizeof(Smem);
    cudaError_t err = cudaFuncSetAttribute(chunk_simt_kernel<T>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    const dim3 grid((unsigned)(a.Hv * (kHeadDim / DVS)), (unsigned)a.B);
    chunk_simt_kernel<T><<<grid, NT, smem, stream>>>(
        (const T *)a.q, (const T *)a.k, (const T *)a.v, a.alpha, a.beta, a.S0, (T *)a.o,
        a.S_final, a.T, a.Hqk, a.Hv, a.cu_seqlens);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_simt(const ChunkArgs &a, gdn_dtype dtype, cudaStream_t stream)
{
    return dtype == GDN_BF16 ? launch_typed<__nv_bfloat16>(a, stream) : launch_typed<float>(a, stream);
}

}  // namespace gdn
