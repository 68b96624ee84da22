// Backward pass: gradients of every input of the gated delta rule.
//
// Forward ("Qwen3.8-Flash-Next 技术总结 -- Qwen4 架构的探路者", section 2.1 "Gated
// DeltaNet", second form of the update), per (sequence, V head):
//   S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,   o_t = S_t^T q_t.
// Its reverse-mode derivative for L = sum_t <dO_t, o_t> + <dS_final, S_T>, walking t
// down with G the gradient with respect to S_t (G = dS_final before the walk):
//   G += q_t dO_t^T;  x = G^T k_t;  w = S_{t-1}^T k_t;  r = v_t - alpha_t w
//   dq_t += S_t dO_t;  dk_t += beta_t G r - alpha_t beta_t S_{t-1} x;  dv_t = beta_t x
//   dbeta_t = x . r;  dalpha_t = <G, S_{t-1}> - beta_t x . w
//   G = alpha_t (G - beta_t k_t x^T)   (then the gradient with respect to S_{t-1});
// dS0 = G after t = 0.
//
// Columns of S (the value dimension) evolve independently in both directions, so
// a CTA owns kCols = 32 columns of one (sequence, V head): 128 threads, thread d
// holds row d of those columns of S (or G) in registers.  Row sums (dq, dk) stay
// in one thread; column sums (S^T k, G^T k) reduce across the CTA (a transposing
// warp reduction, then four warp partials through shared memory).
//   pass 1: the forward, storing S every kCk tokens (checkpoints, workspace);
//   pass 2: blocks of kCk tokens from the end: the block's kCk states are
//           recomputed from its checkpoint into a per-CTA scratch (L2-sized),
//           then its tokens are walked backwards.
// Inputs move a block at a time: the next block's are loaded into registers
// while the current one (staged in shared memory) is processed.
// dq and dk of a QK head sum over its V heads and the four column blocks, dalpha
// and dbeta over the column blocks: fp32 atomic adds into outputs the launcher
// zeroes.  dv and dS0 are written once per element.
#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int kBwdThreads = 128;             // one thread per key dimension d
constexpr int kCols = 32;                    // value columns per CTA
constexpr int kColBlocks = kHeadDim / kCols;
constexpr int kCk = 16;                      // tokens per checkpoint / recompute block
constexpr size_t kSlab = (size_t)kHeadDim * kCols;   // floats of one stored state slice

// Lane l receives the sum over the warp of a[l] (a: 32 values per lane).
__device__ __forceinline__ float warp_transpose_sum(float *a, int lane)
{
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < o; ++i) {
            const float send = up ? a[i] : a[i + o];
            const float keep = up ? a[i + o] : a[i];
            a[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
    return a[0];
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ void store_row(float *dst, const float *x)
{
#pragma unroll
    for (int c = 0; c < kCols; c += 4)
        *reinterpret_cast<float4 *>(dst + c) = make_float4(x[c], x[c + 1], x[c + 2], x[c + 3]);
}
__device__ __forceinline__ void load_row(const float *src, float *x)
{
#pragma unroll
    for (int c = 0; c < kCols; c += 4) {
        const float4 v = *reinterpret_cast<const float4 *>(src + c);
        x[c] = v.x; x[c + 1] = v.y; x[c + 2] = v.z; x[c + 3] = v.w;
    }
}

template <typename T>
struct BwdArgs {
    const T *q, *k, *v, *dO;
    const float *alpha, *beta, *S0, *dS_final;
    float *dq, *dk, *dv, *dalpha, *dbeta, *dS0;
    float *work;
    int T_, Hqk, Hv, nck;
};

// A block of kCk tokens' inputs, staged in shared memory (fp32): k and q of the
// QK head, v and dO at this CTA's columns, the gates.  Tokens past the end hold
// zeros (never used).
struct Block {
    float k[kCk][kHeadDim], q[kCk][kHeadDim];
    float v[kCk][kCols], dO[kCk][kCols];
    float a[kCk], be[kCk];
};

// One thread's share of a block, loaded ahead into registers: its own k, q
// element of every token, a 4-wide piece of v and dO, and one gate value.
struct BlockRegs {
    float k[kCk], q[kCk];
    float4 v, dO;
    float g;
};

template <typename T, bool kBack>
__device__ __forceinline__ void load_block(const BwdArgs<T> &A, int b, int h, int hq, int j0, int t0, int d,
                                           BlockRegs &R)
{
    const int n = min(kCk, A.T_ - t0);
#pragma unroll
    for (int i = 0; i < kCk; ++i) {
        const size_t qk = (((size_t)b * A.T_ + t0 + i) * A.Hqk + hq) * kHeadDim + d;
        R.k[i] = i < n ? to_f32(A.k[qk]) : 0.f;
        R.q[i] = (kBack && i < n) ? to_f32(A.q[qk]) : 0.f;
    }
    const int i = d >> 3, c4 = (d & 7) * 4;             // v, dO: token i, columns c4..c4+3
    R.v = R.dO = make_float4(0.f, 0.f, 0.f, 0.f);
    if (i < n) {
        const size_t off = (((size_t)b * A.T_ + t0 + i) * A.Hv + h) * kHeadDim + j0 + c4;
        R.v = make_float4(to_f32(A.v[off]), to_f32(A.v[off + 1]), to_f32(A.v[off + 2]), to_f32(A.v[off + 3]));
        if (kBack)
            R.dO = make_float4(to_f32(A.dO[off]), to_f32(A.dO[off + 1]), to_f32(A.dO[off + 2]),
                               to_f32(A.dO[off + 3]));
    }
    const int gi = d & (kCk - 1);                        // threads 0-15: alpha, 16-31: beta
    R.g = 0.f;
    if (d < 2 * kCk && gi < n) {
        const size_t g = ((size_t)b * A.T_ + t0 + gi) * A.Hv + h;
        R.g = d < kCk ? A.alpha[g] : A.beta[g];
    }
}

__device__ __forceinline__ void store_block(Block &B, const BlockRegs &R, int d)
{
#pragma unroll
    for (int i = 0; i < kCk; ++i) {
        B.k[i][d] = R.k[i];
        B.q[i][d] = R.q[i];
    }
    const int i = d >> 3, c4 = (d & 7) * 4;
    *reinterpret_cast<float4 *>(&B.v[i][c4]) = R.v;
    *reinterpret_cast<float4 *>(&B.dO[i][c4]) = R.dO;
    if (d < kCk) B.a[d] = R.g;
    else if (d < 2 * kCk) B.be[d - kCk] = R.g;
}

template <typename T>
__global__ void __launch_bounds__(kBwdThreads)
bwd_kernel(const BwdArgs<T> A)
{
    __shared__ __align__(16) Block blk;
    __shared__ __align__(16) float s_red[2][4][kCols];   // warp partials: w, x
    __shared__ __align__(16) float s_tot[2][kCols];      // column sums: w, x
    // warp partials of <G, S_{t-1}>, by token parity: thread 0 reads them after the
    // step's last barrier, when the other warps may already write the next token's
    __shared__ float s_dot[2][4];

    const int jb = blockIdx.x % kColBlocks, h = blockIdx.x / kColBlocks, b = blockIdx.y;
    const int hq = h / (A.Hv / A.Hqk), j0 = jb * kCols;
    const int d = threadIdx.x, lane = d & 31, warp = d >> 5;
    const int nT = A.T_;
    const int nblk = (nT + kCk - 1) / kCk;
    const size_t hs = (size_t)kHeadDim * kHeadDim;
    // this CTA's slice of the workspace: nck checkpoints, then kCk scratch states;
    // thread d only ever stores and reloads row d, so no barrier guards them
    float *ck = A.work + ((((size_t)b * A.Hv + h) * kColBlocks + jb) * (A.nck + kCk)) * kSlab;
    float *scr = ck + (size_t)A.nck * kSlab;

    float S[kCols];
    {
        const float *s0 = A.S0 ? A.S0 + ((size_t)b * A.Hv + h) * hs + (size_t)d * kHeadDim + j0 : nullptr;
#pragma unroll
        for (int c = 0; c < kCols; ++c) S[c] = s0 ? s0[c] : 0.f;
    }

    // One forward step on S with token i of the staged block; `store` (if not
    // null) receives S before the step.
    auto fwd_step = [&](int i, float *store) {
        if (store) store_row(store + (size_t)d * kCols, S);
        const float kd = blk.k[i][d];
        float p[kCols];
#pragma unroll
        for (int c = 0; c < kCols; ++c) p[c] = kd * S[c];
        s_red[0][warp][lane] = warp_transpose_sum(p, lane);
        __syncthreads();
        if (warp == 0)
            s_tot[0][lane] = s_red[0][0][lane] + s_red[0][1][lane] + s_red[0][2][lane] + s_red[0][3][lane];
        __syncthreads();
        const float a = blk.a[i], bk = blk.be[i] * kd;
#pragma unroll
        for (int c = 0; c < kCols; c += 4) {
            const float4 w = *reinterpret_cast<const float4 *>(&s_tot[0][c]);
            const float4 v = *reinterpret_cast<const float4 *>(&blk.v[i][c]);
            S[c] = a * (S[c] - bk * w.x) + bk * v.x;
            S[c + 1] = a * (S[c + 1] - bk * w.y) + bk * v.y;
            S[c + 2] = a * (S[c + 2] - bk * w.z) + bk * v.z;
            S[c + 3] = a * (S[c + 3] - bk * w.w) + bk * v.w;
        }
    };

    BlockRegs R;
    // ---- pass 1: forward with a checkpoint before every block (q, dO staged too:
    //      the last block staged here is the first one pass 2 needs)
    if (nblk > 0) {
        load_block<T, true>(A, b, h, hq, j0, 0, d, R);
#pragma unroll 1
        for (int m = 0; m < nblk; ++m) {
            __syncthreads();                          // the previous block is no longer read
            store_block(blk, R, d);
            __syncthreads();
            if (m + 1 < nblk) load_block<T, true>(A, b, h, hq, j0, (m + 1) * kCk, d, R);
            store_row(ck + (size_t)m * kSlab + (size_t)d * kCols, S);
            const int n = min(kCk, nT - m * kCk);
#pragma unroll 1
            for (int i = 0; i < n; ++i) fwd_step(i, nullptr);
        }
    }

    // ---- pass 2: backward, one block at a time from the end
    float G[kCols];
    {
        const float *g0 = A.dS_final ? A.dS_final + ((size_t)b * A.Hv + h) * hs + (size_t)d * kHeadDim + j0
                                     : nullptr;
#pragma unroll
        for (int c = 0; c < kCols; ++c) G[c] = g0 ? g0[c] : 0.f;
    }
#pragma unroll 1
    for (int m = nblk - 1; m >= 0; --m) {
        const int t0 = m * kCk, n = min(kCk, nT - t0);
        if (m < nblk - 1) {                           // stage block m (loaded ahead)
            __syncthreads();
            store_block(blk, R, d);
            __syncthreads();
        }
        if (m > 0) load_block<T, true>(A, b, h, hq, j0, (m - 1) * kCk, d, R);
        // recompute the block's states: scratch[i] = S before token t0 + i
        load_row(ck + (size_t)m * kSlab + (size_t)d * kCols, S);
#pragma unroll 1
        for (int i = 0; i + 1 < n; ++i) fwd_step(i, scr + (size_t)i * kSlab);
        store_row(scr + (size_t)(n - 1) * kSlab + (size_t)d * kCols, S);
        // walk the block's tokens backwards; S_{t-1} of the next token is loaded one
        // token ahead
        float P[kCols], Pn[kCols];
#pragma unroll
        for (int c = 0; c < kCols; ++c) P[c] = S[c];  // scratch[n - 1] is the current S
#pragma unroll 1
        for (int i = n - 1; i >= 0; --i) {
            const int t = t0 + i;
            if (i > 0) load_row(scr + (size_t)(i - 1) * kSlab + (size_t)d * kCols, Pn);
            const float kd = blk.k[i][d], qd = blk.q[i][d];
            float dot = 0.f;
            {
                float pw[kCols], px[kCols];
#pragma unroll
                for (int c = 0; c < kCols; c += 4) {
                    const float4 o4 = *reinterpret_cast<const float4 *>(&blk.dO[i][c]);
                    G[c] = fmaf(qd, o4.x, G[c]); G[c + 1] = fmaf(qd, o4.y, G[c + 1]);
                    G[c + 2] = fmaf(qd, o4.z, G[c + 2]); G[c + 3] = fmaf(qd, o4.w, G[c + 3]);
                }
#pragma unroll
                for (int c = 0; c < kCols; ++c) {
                    pw[c] = kd * P[c];
                    px[c] = kd * G[c];
                    dot = fmaf(G[c], P[c], dot);
                }
                s_red[0][warp][lane] = warp_transpose_sum(pw, lane);
                s_red[1][warp][lane] = warp_transpose_sum(px, lane);
                dot = warp_sum(dot);
                if (lane == 0) s_dot[i & 1][warp] = dot;
            }
            __syncthreads();
            if (warp == 0) {
                s_tot[0][lane] = s_red[0][0][lane] + s_red[0][1][lane] + s_red[0][2][lane] + s_red[0][3][lane];
                s_tot[1][lane] = s_red[1][0][lane] + s_red[1][1][lane] + s_red[1][2][lane] + s_red[1][3][lane];
            }
            __syncthreads();
            const float a = blk.a[i], be = blk.be[i], bk = be * kd;
            // row sums of this thread: S_t dO, G r, S_{t-1} x; and x . r, x . w
            float sdo = 0.f, gr = 0.f, px = 0.f, xr = 0.f, xw = 0.f;
#pragma unroll
            for (int c4 = 0; c4 < kCols; c4 += 4) {
                const float4 w4 = *reinterpret_cast<const float4 *>(&s_tot[0][c4]);
                const float4 x4 = *reinterpret_cast<const float4 *>(&s_tot[1][c4]);
                const float4 v4 = *reinterpret_cast<const float4 *>(&blk.v[i][c4]);
                const float4 o4 = *reinterpret_cast<const float4 *>(&blk.dO[i][c4]);
                const float wv[4] = {w4.x, w4.y, w4.z, w4.w}, xv[4] = {x4.x, x4.y, x4.z, x4.w};
                const float vv[4] = {v4.x, v4.y, v4.z, v4.w}, ov[4] = {o4.x, o4.y, o4.z, o4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int c = c4 + e;
                    const float w = wv[e], x = xv[e], v = vv[e];
                    const float st = a * (P[c] - bk * w) + bk * v;   // S_t
                    const float r = v - a * w;
                    sdo = fmaf(st, ov[e], sdo);
                    gr = fmaf(G[c], r, gr);
                    px = fmaf(P[c], x, px);
                    xr = fmaf(x, r, xr);
                    xw = fmaf(x, w, xw);
                    G[c] = a * (G[c] - bk * x);                      // gradient w.r.t. S_{t-1}
                }
            }
            const size_t row = (size_t)b * nT + t;
            const size_t qk = (row * A.Hqk + hq) * kHeadDim + d;
            atomicAdd(A.dq + qk, sdo);
            atomicAdd(A.dk + qk, be * gr - a * be * px);
            const size_t g = row * A.Hv + h;
            if (d < kCols) A.dv[g * kHeadDim + j0 + d] = be * s_tot[1][d];
            if (d == 0) {
                atomicAdd(A.dbeta + g, xr);
                const float *sd = s_dot[i & 1];
                atomicAdd(A.dalpha + g, sd[0] + sd[1] + sd[2] + sd[3] - be * xw);
            }
#pragma unroll
            for (int c = 0; c < kCols; ++c) P[c] = Pn[c];
        }
    }
    float *g_out = A.dS0 + ((size_t)b * A.Hv + h) * hs + (size_t)d * kHeadDim + j0;
#pragma unroll
    for (int c = 0; c < kCols; ++c) g_out[c] = G[c];
}

}  // namespace

size_t bwd_workspace(int B, int T, int Hv)
{
    if (B <= 0 || T <= 0 || Hv <= 0) return 0;
    const size_t nck = (size_t)(T + kCk - 1) / kCk;
    return (size_t)B * Hv * kColBlocks * (nck + kCk) * kSlab * sizeof(float);
}

cudaError_t launch_bwd(const BwdLaunch &L, gdn_dtype dtype, cudaStream_t stream)
{
    const size_t n_qk = (size_t)L.B * L.T * L.Hqk * kHeadDim, n_g = (size_t)L.B * L.T * L.Hv;
    cudaError_t err;
    if (n_g > 0) {   // the atomically accumulated outputs start from zero
        if ((err = cudaMemsetAsync(L.dq, 0, n_qk * sizeof(float), stream)) != cudaSuccess) return err;
        if ((err = cudaMemsetAsync(L.dk, 0, n_qk * sizeof(float), stream)) != cudaSuccess) return err;
        if ((err = cudaMemsetAsync(L.dalpha, 0, n_g * sizeof(float), stream)) != cudaSuccess) return err;
        if ((err = cudaMemsetAsync(L.dbeta, 0, n_g * sizeof(float), stream)) != cudaSuccess) return err;
    }
    const dim3 grid((unsigned)(L.Hv * kColBlocks), (unsigned)L.B);
    const int nck = (L.T + kCk - 1) / kCk;
    if (dtype == GDN_BF16) {
        BwdArgs<__nv_bfloat16> A{(const __nv_bfloat16 *)L.q, (const __nv_bfloat16 *)L.k,
                                 (const __nv_bfloat16 *)L.v, (const __nv_bfloat16 *)L.dO,
                                 L.alpha, L.beta, L.S0, L.dS_final, L.dq, L.dk, L.dv, L.dalpha,
                                 L.dbeta, L.dS0, L.work, L.T, L.Hqk, L.Hv, nck};
        bwd_kernel<__nv_bfloat16><<<grid, kBwdThreads, 0, stream>>>(A);
    } else {
        BwdArgs<float> A{(const float *)L.q, (const float *)L.k, (const float *)L.v, (const float *)L.dO,
                         L.alpha, L.beta, L.S0, L.dS_final, L.dq, L.dk, L.dv, L.dalpha,
                         L.dbeta, L.dS0, L.work, L.T, L.Hqk, L.Hv, nck};
        bwd_kernel<float><<<grid, kBwdThreads, 0, stream>>>(A);
    }
    return cudaGetLastError();
}

}  // namespace gdn
