// Chunkwise (WY) backward pass of the gated delta rule, bf16 inputs.
//
// Forward, per chunk of C = 64 tokens of one (sequence, V head), from the state S at
// the chunk's start ("Qwen3.8-Flash-Next 技术总结 -- Qwen4 架构的探路者", section 2.1
// "Gated DeltaNet": the update S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} +
// beta_t k_t v_t^T evaluated chunk by chunk with the WY representation), with
// b = cumsum(log alpha), gamma = exp(b), Gam[r][i] = exp(b_r - b_i) (i <= r),
// g = exp(b_{C-1} - b), A = strict_lower(diag(beta) (Gam o K K^T)), T = (I + A)^-1:
//   W = T diag(beta gamma) K,  U~ = T diag(beta) V,  U = U~ - W S,  P = Gam o Q K^T
//   O = diag(gamma) Q S + P U,  S' = gamma_{C-1} S + K^T diag(g) U.
// The backward is the chain rule through these equations, chunk by chunk from the
// end, given dO and dS' (the gradient of the chunk's end state):
//   dU = diag(g) K dS' + P^T dO,   dS = gamma_{C-1} dS' + Q^T diag(gamma) dO - W^T dU
// (the serial part), then per chunk, independently of the others:
//   dQ = diag(gamma) dO S^T + (dP o Gam) K,   dP = dO U^T,   dW = -dU S^T
//   dK = (dP o Gam)^T Q + diag(g) U dS'^T + diag(beta gamma) T^T dW + (M + M^T) K
//   dV = diag(beta) T^T dU,   dT = dW (diag(beta gamma) K)^T + dU (diag(beta) V)^T
//   dA = strict_lower(-T^T dT T^T),   M = diag(beta) (dA o Gam)
// and the gate gradients through beta, gamma, Gam, g and gamma_{C-1} into b, whose
// reverse cumulative sum is d log alpha.  A ragged last chunk is padded with tokens
// that leave the state alone (k = q = v = dO = 0, alpha = 1, beta = 0), which makes
// row C-1 the chunk's last row in every formula.
//
// Four launches, all on warp-level bf16 tensor-core MMAs (m16n8k16, fp32
// accumulation) fed by ldmatrix from padded shared-memory tiles:
//   1. prep_kernel, per (chunk, QK head): grams, the triangular solve (fp32), and
//      per V head W, U~, T, P and the gate vectors b, gamma, g into the workspace;
//   2. fwd_chain_kernel, per (V head, 64 value columns): the chunk start states S
//      (bf16, kept for step 4) and U = U~ - W S (over U~ in the workspace);
//   3. grad_chain_kernel, per (V head, 64 value columns), chunks from the end: dS'
//      (bf16) and dU per chunk, sum(dS' o S) per chunk, and dS0;
//   4. grad_chunk_kernel, per (chunk, QK head), its V heads in turn: every other
//      gradient, dq and dk summed over the V heads in registers (no atomics: the
//      results do not depend on scheduling).
// Columns of S and dS evolve independently, so the two chains split the value
// dimension over CTAs; the chains are the only serial work.
#include "gdn_internal.cuh"

namespace gdn {
namespace {

using bf16 = __nv_bfloat16;
constexpr int C = kChunk;            // 64 tokens per chunk
constexpr int D = kHeadDim;          // 128
constexpr int LDT = D + 8;           // row stride (elements) of 64 x 128 and 128 x 128 bf16 tiles
constexpr int LDQ = C + 8;           // 64 x 64 bf16 tiles
constexpr int LDF = C + 1;           // 64 x 64 fp32 tiles
constexpr int kThreads = 256;        // 8 warps (grad_chunk_kernel: K3W warps, below)
constexpr float kLogFloor = -87.f;   // log alpha clamp (alpha = 0 stays finite)

// Workspace, per (sequence, V head, chunk) ch = (b Hv + h) NC + n.
struct Ws {
    bf16 *W;       // [ch][64][128]  W
    bf16 *U;       // [ch][64][128]  U~ (prep), then U (forward chain)
    bf16 *Tm;      // [ch][64][64]   T = (I + A)^-1
    bf16 *P;       // [ch][64][64]   Gam o Q K^T
    bf16 *S;       // [ch][128][128] S at the chunk start, [d][j]
    bf16 *dSp;     // [ch][128][128] gradient of the chunk's end state, [d][j]
    bf16 *dU;      // [ch][64][128]  dU
    float *gate;   // [ch][3][64]    b = cumsum(log alpha) inside the chunk, gamma = exp(b),
                   //                g = exp(b_63 - b)
    float *gC;     // [ch][2]        sum(dS' o S) over each 64-column block
};

struct Params {
    const bf16 *q, *k, *v, *dO;
    const float *alpha, *beta, *S0, *dS_final;
    float *dq, *dk, *dv, *dalpha, *dbeta, *dS0;
    Ws ws;
    int B, T, Hqk, Hv, NC;
};

// ------------------------------------------------------------------ warp MMA helpers
__device__ __forceinline__ uint32_t sa(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void ldsm4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr) : "memory");
}
__device__ __forceinline__ void ldsm4t(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr) : "memory");
}
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
                 "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// acc (16 rows from m0, 8 NT columns from n0) += A B over k in [0, K), one warp.
// AL = 0: A stored [m][k]; AL = 1: A stored [k][m] (the product uses A^T of the tile).
// BL = 0: B stored [n][k]; BL = 1: B stored [k][n].  lda, ldb in elements; every row
// of a tile starts on a 16-byte boundary.
// Fragment layout of acc[nt][e]: row m0 + (lane >> 2) + 8 (e >> 1), column
// n0 + 8 nt + 2 (lane & 3) + (e & 1).
template <int AL, int BL, int NT, int UNROLL = 8>
__device__ __forceinline__ void warp_mma(float (&acc)[NT][4], const bf16 *A, int lda, const bf16 *Bm,
                                         int ldb, int m0, int n0, int K, int lane)
{
    static_assert(NT % 2 == 0, "n tiles in pairs");
#pragma unroll UNROLL
    for (int k0 = 0; k0 < K; k0 += 16) {
        uint32_t a[4];
        if (AL == 0)
            ldsm4(sa(A + (m0 + (lane & 15)) * lda + k0 + 8 * (lane >> 4)), a);
        else
            ldsm4t(sa(A + (k0 + (lane & 7) + 8 * (lane >> 4)) * lda + m0 + 8 * ((lane >> 3) & 1)), a);
#pragma unroll
        for (int nt = 0; nt < NT; nt += 2) {
            uint32_t bb[4];
            const int nb = n0 + 8 * nt;
            if (BL == 0)
                ldsm4(sa(Bm + (nb + (lane & 7) + 8 * (lane >> 4)) * ldb + k0 + 8 * ((lane >> 3) & 1)), bb);
            else
                ldsm4t(sa(Bm + (k0 + (lane & 7) + 8 * ((lane >> 3) & 1)) * ldb + nb + 8 * (lane >> 4)), bb);
            mma16816(acc[nt], a, bb[0], bb[1]);
            mma16816(acc[nt + 1], a, bb[2], bb[3]);
        }
    }
}

__device__ __forceinline__ uint32_t scale_bf16x2(uint32_t v, float lo, float hi) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&v));
    const __nv_bfloat162 h = __floats2bfloat162_rn(f.x * lo, f.y * hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// acc += (diag(ks) A)^T-side product: as warp_mma<1, 1, NT> (A stored [k][m], B stored
// [k][n]) with every A element of index k scaled by ks[k] in the fragment (one bf16
// rounding), so a per-k scale needs no scaled copy of a tile.
template <int NT>
__device__ __forceinline__ void warp_mma_kscaled(float (&acc)[NT][4], const bf16 *A, int lda, const float *ks,
                                                 const bf16 *Bm, int ldb, int m0, int n0, int K, int lane)
{
    static_assert(NT % 2 == 0, "n tiles in pairs");
    const int t2 = 2 * (lane & 3);
#pragma unroll 8
    for (int k0 = 0; k0 < K; k0 += 16) {
        uint32_t a[4];
        ldsm4t(sa(A + (k0 + (lane & 7) + 8 * (lane >> 4)) * lda + m0 + 8 * ((lane >> 3) & 1)), a);
        const float s0 = ks[k0 + t2], s1 = ks[k0 + t2 + 1], s2 = ks[k0 + 8 + t2], s3 = ks[k0 + 9 + t2];
        a[0] = scale_bf16x2(a[0], s0, s1);
        a[1] = scale_bf16x2(a[1], s0, s1);
        a[2] = scale_bf16x2(a[2], s2, s3);
        a[3] = scale_bf16x2(a[3], s2, s3);
#pragma unroll
        for (int nt = 0; nt < NT; nt += 2) {
            uint32_t bb[4];
            const int nb = n0 + 8 * nt;
            ldsm4t(sa(Bm + (k0 + (lane & 7) + 8 * ((lane >> 3) & 1)) * ldb + nb + 8 * (lane >> 4)), bb);
            mma16816(acc[nt], a, bb[0], bb[1]);
            mma16816(acc[nt + 1], a, bb[2], bb[3]);
        }
    }
}

template <int NT>
__device__ __forceinline__ void zero_acc(float (&acc)[NT][4]) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}
__device__ __forceinline__ float2 unpack2(const bf16 *p) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(p));
}

// ------------------------------------------------------------------ async tile loads
__device__ __forceinline__ void cp16(void *dst, const void *src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;"
                 ::"r"(sa(dst)), "l"(src), "r"(valid ? 16 : 0) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// ROWS x (8 NCH) bf16 from src (row r at src + r * src_ld) into dst (row stride ld);
// rows >= valid_rows are zero-filled without being read.
template <int ROWS, int NCH, int NTHR = kThreads>
__device__ __forceinline__ void load_tile(bf16 *dst, int ld, const bf16 *src, size_t src_ld, int valid_rows,
                                          int tid)
{
#pragma unroll 4
    for (int e = tid; e < ROWS * NCH; e += NTHR) {
        const int r = e / NCH, c = e % NCH;
        const bool ok = r < valid_rows;
        cp16(dst + r * ld + 8 * c, src + (size_t)(ok ? r : 0) * src_ld + 8 * c, ok);
    }
}

// The 192 gate floats of a chunk (768 bytes) by 48 cp.async of 16 bytes.
__device__ __forceinline__ void load_gate(float *dst, const float *src, int tid) {
    if (tid < 48) cp16(dst + 4 * tid, src + 4 * tid, true);
}

// K K^T and Q K^T of one chunk (64 x 64, fp32) from the bf16 tiles, in the warp
// tiling of grad_chunk_kernel (K3W warps, warp tile 16 x 64 / (K3W / 4)).
constexpr int K3W = 16;                  // warps of grad_chunk_kernel
constexpr int K3T = 32 * K3W;
constexpr int K3H = K3W / 4;             // warps sharing a 16-row block
constexpr int NTA = 128 / K3H / 8;       // n tiles of a 64 x 128 product per warp
constexpr int NTB = 64 / K3H / 8;        // n tiles of a 64 x 64 product per warp
__device__ __forceinline__ void chunk_grams(const bf16 *sK, const bf16 *sQ, float *fKK, float *fQK, int warp,
                                            int lane)
{
    const int m0 = 16 * (warp & 3), n0 = 8 * NTB * (warp >> 2);
    float kk[NTB][4], qk[NTB][4];
    zero_acc(kk);
    zero_acc(qk);
    warp_mma<0, 0, NTB>(kk, sK, LDT, sK, LDT, m0, n0, D, lane);
    warp_mma<0, 0, NTB>(qk, sQ, LDT, sK, LDT, m0, n0, D, lane);
#pragma unroll
    for (int nt = 0; nt < NTB; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int r = m0 + (lane >> 2) + 8 * (e >> 1), s = n0 + 8 * nt + 2 * (lane & 3) + (e & 1);
            fKK[r * LDF + s] = kk[nt][e];
            fQK[r * LDF + s] = qk[nt][e];
        }
}

// T = (I + A)^-1 for the strictly lower 64 x 64 A (fp32, row stride LDF), in place,
// by 16 x 16 blocks: the diagonal blocks by forward substitution (one thread per
// column, the column in registers until every thread has read its block of A),
// then block rows 1..3 in turn,
//   T_ij = -T_ii sum_{j <= k < i} A_ik T_kj   (j < i),
// every element of a stage in parallel: block row i still holds A while its X_ij
// are formed, and the rows above it already hold T.  The upper blocks of A are
// zero, as T's are.  xs: 768 floats of scratch.  Called by all threads; ends with
// the result visible.
__device__ __forceinline__ void invert_unit_lower(float *fAT, float *xs, int tid)
{
    float t[16];
    const int base = 16 * (tid >> 4), c = tid & 15;
    if (tid < 64) {
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float s = r == c ? 1.f : 0.f;
#pragma unroll
            for (int m = 0; m < r; ++m) s -= fAT[(base + r) * LDF + base + m] * t[m];
            t[r] = r < c ? 0.f : s;
        }
    }
    __syncthreads();   // every diagonal block of A read
    if (tid < 64) {
#pragma unroll
        for (int r = 0; r < 16; ++r) fAT[(base + r) * LDF + base + c] = t[r];
    }
    __syncthreads();
    for (int i = 1; i < 4; ++i) {
        for (int e = tid; e < i * 256; e += kThreads) {
            const int j = e >> 8, r = (e >> 4) & 15, cc = e & 15;
            float s = 0.f;
            for (int k = j; k < i; ++k)
#pragma unroll
                for (int m = 0; m < 16; ++m)
                    s += fAT[(16 * i + r) * LDF + 16 * k + m] * fAT[(16 * k + m) * LDF + 16 * j + cc];
            xs[e] = s;
        }
        __syncthreads();
        for (int e = tid; e < i * 256; e += kThreads) {
            const int j = e >> 8, r = (e >> 4) & 15, cc = e & 15;
            float s = 0.f;
#pragma unroll
            for (int m = 0; m < 16; ++m) s += fAT[(16 * i + r) * LDF + 16 * i + m] * xs[(j << 8) + (m << 4) + cc];
            fAT[(16 * i + r) * LDF + 16 * j + cc] = -s;
        }
        __syncthreads();
    }
}

// ================================================================== 1. preparation
// Per (chunk n, QK head hq, sequence b): grams once (K K^T fp32, Q K^T bf16), then
// for each V head of the group the decay vectors, A, the solve T = (I + A)^-1 (fp32,
// blocked, in place), P = Gam o Q K^T, and W = (T diag(beta gamma)) K,
// U~ = (T diag(beta)) V with the gates folded into the columns of T; all to the
// workspace.  111 KB of shared memory: two CTAs per SM.
constexpr size_t P_K = 0;
constexpr size_t P_Q = P_K + 64 * LDT * 2;
constexpr size_t P_V = P_Q + 64 * LDT * 2;
constexpr size_t P_TW = P_V + 64 * LDT * 2;     // T diag(beta gamma), bf16 (the solve's scratch before)
constexpr size_t P_TU = P_TW + 64 * LDQ * 2;    // T diag(beta), bf16
constexpr size_t P_QK = P_TU + 64 * LDQ * 2;    // Q K^T, bf16
constexpr size_t P_KK = P_QK + 64 * LDQ * 2;    // K K^T, fp32
constexpr size_t P_AT = P_KK + 64 * LDF * 4;    // A, then T (fp32)
constexpr size_t P_G = P_AT + 64 * LDF * 4;     // b[64], beta[64], gamma[64]
constexpr size_t P_BYTES = P_G + 3 * 64 * 4;

__global__ void __launch_bounds__(kThreads, 2) prep_kernel(const Params p)
{
    extern __shared__ __align__(128) unsigned char smem[];
    bf16 *sK = reinterpret_cast<bf16 *>(smem + P_K), *sQ = reinterpret_cast<bf16 *>(smem + P_Q);
    bf16 *sV = reinterpret_cast<bf16 *>(smem + P_V);
    bf16 *sTw = reinterpret_cast<bf16 *>(smem + P_TW), *sTu = reinterpret_cast<bf16 *>(smem + P_TU);
    bf16 *sQK = reinterpret_cast<bf16 *>(smem + P_QK);
    float *fKK = reinterpret_cast<float *>(smem + P_KK), *fAT = reinterpret_cast<float *>(smem + P_AT);
    float *sb = reinterpret_cast<float *>(smem + P_G), *sbeta = sb + 64, *sgam = sb + 128;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n = blockIdx.x, hq = blockIdx.y, b = blockIdx.z;
    const int grp = p.Hv / p.Hqk;
    const int t0 = n * C, L = min(C, p.T - t0);
    const size_t qk_ld = (size_t)p.Hqk * D, v_ld = (size_t)p.Hv * D;
    load_tile<64, 16>(sK, LDT, p.k + ((size_t)b * p.T + t0) * qk_ld + (size_t)hq * D, qk_ld, L, tid);
    load_tile<64, 16>(sQ, LDT, p.q + ((size_t)b * p.T + t0) * qk_ld + (size_t)hq * D, qk_ld, L, tid);
    cp_commit();
    load_tile<64, 16>(sV, LDT, p.v + ((size_t)b * p.T + t0) * v_ld + (size_t)(hq * grp) * D, v_ld, L, tid);
    cp_commit();
    cp_wait<1>();
    __syncthreads();
    {   // K K^T (fp32) and Q K^T (bf16): 64 x 64, warp tile 16 x 32
        const int m0 = 16 * (warp & 3), n0 = 32 * (warp >> 2);
        float kk[4][4], qk[4][4];
        zero_acc(kk);
        zero_acc(qk);
        warp_mma<0, 0, 4>(kk, sK, LDT, sK, LDT, m0, n0, D, lane);
        warp_mma<0, 0, 4>(qk, sQ, LDT, sK, LDT, m0, n0, D, lane);
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const int r = m0 + (lane >> 2) + 8 * hf, c = n0 + 8 * nt + 2 * (lane & 3);
                fKK[r * LDF + c] = kk[nt][2 * hf];
                fKK[r * LDF + c + 1] = kk[nt][2 * hf + 1];
                *reinterpret_cast<uint32_t *>(sQK + r * LDQ + c) = pack2(qk[nt][2 * hf], qk[nt][2 * hf + 1]);
            }
    }
    for (int i = 0; i < grp; ++i) {
        const int h = hq * grp + i;
        const size_t ch = ((size_t)b * p.Hv + h) * p.NC + n;
        __syncthreads();   // grams written; the previous head's tiles no longer read
        if (i > 0) {
            load_tile<64, 16>(sV, LDT, p.v + ((size_t)b * p.T + t0) * v_ld + (size_t)h * D, v_ld, L, tid);
            cp_commit();
        }
        if (warp == 0) {   // b = cumsum(log alpha), two rows per lane; padded rows add 0
            const float *al = p.alpha + ((size_t)b * p.T + t0) * p.Hv + h;
            const float *be = p.beta + ((size_t)b * p.T + t0) * p.Hv + h;
            const int r0 = 2 * lane, r1 = r0 + 1;
            const float l0 = r0 < L ? fmaxf(logf(al[(size_t)r0 * p.Hv]), kLogFloor) : 0.f;
            const float l1 = r1 < L ? fmaxf(logf(al[(size_t)r1 * p.Hv]), kLogFloor) : 0.f;
            float s = l0 + l1;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, s, o);
                if (lane >= o) s += y;
            }
            const float excl = s - (l0 + l1);
            const float blast = __shfl_sync(0xffffffffu, s, 31);
            const float b0 = excl + l0, b1 = excl + l0 + l1;
            sb[r0] = b0;
            sb[r1] = b1;
            sbeta[r0] = r0 < L ? be[(size_t)r0 * p.Hv] : 0.f;
            sbeta[r1] = r1 < L ? be[(size_t)r1 * p.Hv] : 0.f;
            const float ga0 = expf(b0), ga1 = expf(b1);
            sgam[r0] = ga0;
            sgam[r1] = ga1;
            float *gv = p.ws.gate + ch * 192;
            *reinterpret_cast<float2 *>(gv + r0) = make_float2(b0, b1);
            *reinterpret_cast<float2 *>(gv + 64 + r0) = make_float2(ga0, ga1);
            *reinterpret_cast<float2 *>(gv + 128 + r0) = make_float2(expf(blast - b0), expf(blast - b1));
        }
        __syncthreads();
        // Gam[r][m] = exp(b_r - b_m) once per lower element: A[r][m] = beta_r Gam KK (m < r),
        // P[r][m] = Gam QK (m <= r) -> workspace
        {
            bf16 *gP = p.ws.P + ch * 64 * 64;
            for (int e = tid; e < 64 * 32; e += kThreads) {
                const int r = e >> 5, m2 = 2 * (e & 31);
                const float2 qk2 = unpack2(sQK + r * LDQ + m2);
                const float qkv[2] = {qk2.x, qk2.y};
                float pv[2];
#pragma unroll
                for (int x = 0; x < 2; ++x) {
                    const int m = m2 + x;
                    const float gam = m <= r ? __expf(sb[r] - sb[m]) : 0.f;
                    fAT[r * LDF + m] = m < r ? sbeta[r] * gam * fKK[r * LDF + m] : 0.f;
                    pv[x] = gam * qkv[x];
                }
                *reinterpret_cast<uint32_t *>(gP + r * 64 + m2) = pack2(pv[0], pv[1]);
            }
        }
        __syncthreads();
        invert_unit_lower(fAT, reinterpret_cast<float *>(sTw), tid);   // sTw is free until below
        // T -> workspace (bf16); T diag(beta gamma), T diag(beta) -> tiles
        {
            bf16 *gT = p.ws.Tm + ch * 64 * 64;
            for (int e = tid; e < 64 * 32; e += kThreads) {
                const int r = e >> 5, c2 = 2 * (e & 31);
                const float ta = fAT[r * LDF + c2], tb = fAT[r * LDF + c2 + 1];
                *reinterpret_cast<uint32_t *>(gT + r * 64 + c2) = pack2(ta, tb);
                *reinterpret_cast<uint32_t *>(sTw + r * LDQ + c2) =
                    pack2(ta * sbeta[c2] * sgam[c2], tb * sbeta[c2 + 1] * sgam[c2 + 1]);
                *reinterpret_cast<uint32_t *>(sTu + r * LDQ + c2) = pack2(ta * sbeta[c2], tb * sbeta[c2 + 1]);
            }
        }
        cp_wait_all();
        __syncthreads();   // V landed; the scaled T tiles complete
        // W = (T diag(beta gamma)) K, U~ = (T diag(beta)) V: 64 x 128, K = 64
        {
            const int m0 = 16 * (warp & 3), n0 = 64 * (warp >> 2);
            float acc[8][4];
            bf16 *gW = p.ws.W + ch * 64 * D, *gU = p.ws.U + ch * 64 * D;
#pragma unroll 1
            for (int which = 0; which < 2; ++which) {
                zero_acc(acc);
                warp_mma<0, 1, 8>(acc, which ? sTu : sTw, LDQ, which ? sV : sK, LDT, m0, n0, C, lane);
                bf16 *dst = which ? gU : gW;
#pragma unroll
                for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        const int r = m0 + (lane >> 2) + 8 * hf, c = n0 + 8 * nt + 2 * (lane & 3);
                        *reinterpret_cast<uint32_t *>(dst + r * D + c) = pack2(acc[nt][2 * hf], acc[nt][2 * hf + 1]);
                    }
            }
        }
    }
}

// ================================================================== 2. forward chain
// Per (FJ-column block, V head h, sequence b): S (128 x FJ fp32, mma accumulators,
// warp w rows 16w..16w+15) from S0, then per chunk: S -> workspace (bf16),
// U = U~ - W S -> workspace, S <- gamma_{C-1} S + K^T diag(g) U.  A two-stage ring
// holds each chunk's W, K, U~ block and decay, loaded one whole chunk ahead, so the
// serial path never waits for memory.
constexpr int FJ = 64;                          // value columns per CTA (one CTA per SM at B=1, 48 heads)
constexpr int FLDJ = FJ + 8;
constexpr size_t FS_W = 0;                      // one ring stage
constexpr size_t FS_K = FS_W + 64 * LDT * 2;
constexpr size_t FS_UT = FS_K + 64 * LDT * 2;   // U~ block, 64 x FJ
constexpr size_t FS_GB = FS_UT + 64 * FLDJ * 2; // gates: b, gamma, g (64 each)
constexpr size_t FS_BYTES = FS_GB + 192 * 4;
constexpr size_t F_S = 2 * FS_BYTES;            // S block, bf16, 128 x FJ ([d][j])
constexpr size_t F_U = F_S + 128 * FLDJ * 2;    // diag(g) U block, bf16
constexpr size_t F_BYTES = F_U + 64 * FLDJ * 2;

constexpr int FNT = FJ / 8;                     // n tiles of the state block per warp

__global__ void __launch_bounds__(kThreads, FJ == 32 ? 2 : 1) fwd_chain_kernel(const Params p)
{
    extern __shared__ __align__(128) unsigned char smem[];
    bf16 *sS = reinterpret_cast<bf16 *>(smem + F_S), *sU = reinterpret_cast<bf16 *>(smem + F_U);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int j0 = FJ * blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int hq = h / (p.Hv / p.Hqk);
    const size_t qk_ld = (size_t)p.Hqk * D;
    const size_t ch0 = ((size_t)b * p.Hv + h) * p.NC;
    float s[FNT][4];   // S rows 16 warp + (lane >> 2) (+8), columns 8 nt + 2 (lane & 3) (+1)
#pragma unroll
    for (int nt = 0; nt < FNT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int r = 16 * warp + (lane >> 2) + 8 * (e >> 1), c = 8 * nt + 2 * (lane & 3) + (e & 1);
            s[nt][e] = p.S0 ? p.S0[((size_t)b * p.Hv + h) * D * D + (size_t)r * D + j0 + c] : 0.f;
        }
    auto load = [&](int n) {
        unsigned char *st = smem + (n & 1) * FS_BYTES;
        load_tile<64, 16>(reinterpret_cast<bf16 *>(st + FS_W), LDT, p.ws.W + (ch0 + n) * 64 * D, D, 64, tid);
        load_tile<64, 16>(reinterpret_cast<bf16 *>(st + FS_K), LDT,
                          p.k + ((size_t)b * p.T + n * C) * qk_ld + (size_t)hq * D, qk_ld,
                          min(C, p.T - n * C), tid);
        load_tile<64, FJ / 8>(reinterpret_cast<bf16 *>(st + FS_UT), FLDJ, p.ws.U + (ch0 + n) * 64 * D + j0, D,
                              64, tid);
        load_gate(reinterpret_cast<float *>(st + FS_GB), p.ws.gate + (ch0 + n) * 192, tid);
        cp_commit();
    };
    load(0);
    if (p.NC > 1) load(1);
    for (int n = 0; n < p.NC; ++n) {
        const size_t ch = ch0 + n;
        const unsigned char *st = smem + (n & 1) * FS_BYTES;
        const bf16 *sW = reinterpret_cast<const bf16 *>(st + FS_W), *sK = reinterpret_cast<const bf16 *>(st + FS_K);
        const bf16 *sUt = reinterpret_cast<const bf16 *>(st + FS_UT);
        const float *sgb = reinterpret_cast<const float *>(st + FS_GB);
        // S at the chunk start -> bf16 tile and workspace
        bf16 *gS = p.ws.S + ch * D * D + j0;
#pragma unroll
        for (int nt = 0; nt < FNT; ++nt)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const int r = 16 * warp + (lane >> 2) + 8 * hf, c = 8 * nt + 2 * (lane & 3);
                const uint32_t v2 = pack2(s[nt][2 * hf], s[nt][2 * hf + 1]);
                *reinterpret_cast<uint32_t *>(sS + r * FLDJ + c) = v2;
                *reinterpret_cast<uint32_t *>(gS + (size_t)r * D + c) = v2;
            }
        if (n + 1 < p.NC) cp_wait<1>(); else cp_wait<0>();
        __syncthreads();   // stage n landed; S tile complete
        const float glast = sgb[64 + 63];
        // U = U~ - W S: 64 x FJ, warp tile 16 x FJ/2
        {
            const int m0 = 16 * (warp & 3), n0 = (FJ / 2) * (warp >> 2);
            float u[FNT / 2][4];
            zero_acc(u);
            warp_mma<0, 1, FNT / 2>(u, sW, LDT, sS, FLDJ, m0, n0, D, lane);
            bf16 *gU = p.ws.U + ch * 64 * D + j0;
#pragma unroll
            for (int nt = 0; nt < FNT / 2; ++nt)
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const int r = m0 + (lane >> 2) + 8 * hf, c = n0 + 8 * nt + 2 * (lane & 3);
                    const float2 ut = unpack2(sUt + r * FLDJ + c);
                    const float u0 = ut.x - u[nt][2 * hf], u1 = ut.y - u[nt][2 * hf + 1];
                    const float gr = sgb[128 + r];
                    *reinterpret_cast<uint32_t *>(gU + (size_t)r * D + c) = pack2(u0, u1);
                    *reinterpret_cast<uint32_t *>(sU + r * FLDJ + c) = pack2(gr * u0, gr * u1);
                }
        }
        __syncthreads();   // diag(g) U complete
        // S <- gamma_{C-1} S + K^T diag(g) U: 128 x FJ, warp tile 16 x FJ, K = 64
#pragma unroll
        for (int nt = 0; nt < FNT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) s[nt][e] *= glast;
        warp_mma<1, 1, FNT>(s, sK, LDT, sU, FLDJ, 16 * warp, 0, C, lane);
        __syncthreads();   // stage n, S tile and U tile no longer read
        if (n + 2 < p.NC) load(n + 2);
    }
}

// ================================================================== 3. gradient chain
// Per (64-column block jb, V head h, sequence b), chunks from the last: dS (128 x 64
// fp32 accumulators, warp w rows 16w..16w+15) from dS_final; per chunk: dS' = dS ->
// workspace (bf16), dU = diag(g) K dS' + P^T dO -> workspace, sum(dS' o S) -> gC,
// dS <- gamma_{C-1} dS' + Q^T diag(gamma) dO - W^T dU.  At the end dS0 = dS.  A
// two-stage ring holds each chunk's K, Q, W, P, dO block, start-state block and
// decay, loaded one whole chunk ahead.
constexpr int GJ = 64;                          // value columns per CTA
constexpr int GLDJ = GJ + 8;
constexpr int kGcSlots = D / GJ;                // partial sums of sum(dS' o S) per chunk
constexpr size_t GS_K = 0;                      // one ring stage
constexpr size_t GS_Q = GS_K + 64 * LDT * 2;
constexpr size_t GS_W = GS_Q + 64 * LDT * 2;
constexpr size_t GS_P = GS_W + 64 * LDT * 2;    // P, 64 x 64
constexpr size_t GS_O = GS_P + 64 * LDQ * 2;    // dO block, 64 x 64
constexpr size_t GS_SB = GS_O + 64 * GLDJ * 2;  // S block at the chunk start, 128 x 64
constexpr size_t GS_GB = GS_SB + 128 * GLDJ * 2;
constexpr size_t GS_BYTES = GS_GB + 192 * 4;
constexpr size_t G_D = 2 * GS_BYTES;            // dS' block, bf16, 128 x 64
constexpr size_t G_DU = G_D + 128 * GLDJ * 2;   // -dU block
constexpr size_t G_PART = G_DU + 64 * GLDJ * 2; // partial sums[8]
constexpr size_t G_BYTES = G_PART + 8 * 4;

__global__ void __launch_bounds__(kThreads, 1) grad_chain_kernel(const Params p)
{
    extern __shared__ __align__(128) unsigned char smem[];
    bf16 *sD = reinterpret_cast<bf16 *>(smem + G_D);
    bf16 *sdU = reinterpret_cast<bf16 *>(smem + G_DU);
    float *spart = reinterpret_cast<float *>(smem + G_PART);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int jb = blockIdx.x, j0 = GJ * jb, h = blockIdx.y, b = blockIdx.z;
    const int hq = h / (p.Hv / p.Hqk);
    const size_t qk_ld = (size_t)p.Hqk * D, v_ld = (size_t)p.Hv * D;
    const size_t ch0 = ((size_t)b * p.Hv + h) * p.NC;
    const size_t hs = ((size_t)b * p.Hv + h) * D * D;
    float ds[8][4];   // rows 16 warp + (lane >> 2) (+8), columns 8 nt + 2 (lane & 3) (+1)
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int r = 16 * warp + (lane >> 2) + 8 * (e >> 1), c = 8 * nt + 2 * (lane & 3) + (e & 1);
            ds[nt][e] = p.dS_final ? p.dS_final[hs + (size_t)r * D + j0 + c] : 0.f;
        }
    auto load = [&](int n) {
        unsigned char *st = smem + (n & 1) * GS_BYTES;
        const int L = min(C, p.T - n * C);
        const size_t tok = (size_t)b * p.T + n * C;
        load_tile<64, 16>(reinterpret_cast<bf16 *>(st + GS_K), LDT, p.k + tok * qk_ld + (size_t)hq * D, qk_ld, L,
                          tid);
        load_tile<64, 16>(reinterpret_cast<bf16 *>(st + GS_Q), LDT, p.q + tok * qk_ld + (size_t)hq * D, qk_ld, L,
                          tid);
        load_tile<64, 16>(reinterpret_cast<bf16 *>(st + GS_W), LDT, p.ws.W + (ch0 + n) * 64 * D, D, 64, tid);
        load_tile<64, 8>(reinterpret_cast<bf16 *>(st + GS_P), LDQ, p.ws.P + (ch0 + n) * 64 * 64, 64, 64, tid);
        load_tile<64, 8>(reinterpret_cast<bf16 *>(st + GS_O), GLDJ, p.dO + tok * v_ld + (size_t)h * D + j0, v_ld,
                         L, tid);
        load_tile<128, 8>(reinterpret_cast<bf16 *>(st + GS_SB), GLDJ, p.ws.S + (ch0 + n) * D * D + j0, D, 128,
                          tid);
        load_gate(reinterpret_cast<float *>(st + GS_GB), p.ws.gate + (ch0 + n) * 192, tid);
        cp_commit();
    };
    load(p.NC - 1);
    if (p.NC > 1) load(p.NC - 2);
    for (int n = p.NC - 1; n >= 0; --n) {
        const size_t ch = ch0 + n;
        const unsigned char *st = smem + (n & 1) * GS_BYTES;
        const bf16 *sK = reinterpret_cast<const bf16 *>(st + GS_K), *sQ = reinterpret_cast<const bf16 *>(st + GS_Q);
        const bf16 *sW = reinterpret_cast<const bf16 *>(st + GS_W), *sP = reinterpret_cast<const bf16 *>(st + GS_P);
        const bf16 *sO = reinterpret_cast<const bf16 *>(st + GS_O), *sSb = reinterpret_cast<const bf16 *>(st + GS_SB);
        const float *sgb = reinterpret_cast<const float *>(st + GS_GB);
        // dS' -> bf16 tile and workspace
        {
            bf16 *gD = p.ws.dSp + ch * D * D + j0;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const int r = 16 * warp + (lane >> 2) + 8 * hf, c = 8 * nt + 2 * (lane & 3);
                    const uint32_t v2 = pack2(ds[nt][2 * hf], ds[nt][2 * hf + 1]);
                    *reinterpret_cast<uint32_t *>(sD + r * GLDJ + c) = v2;
                    *reinterpret_cast<uint32_t *>(gD + (size_t)r * D + c) = v2;
                }
        }
        if (n >= 1) cp_wait<1>(); else cp_wait<0>();
        __syncthreads();   // stage n landed; dS' tile complete
        {   // sum(dS' o S) over this block
            float gc = 0.f;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const int r = 16 * warp + (lane >> 2) + 8 * hf, c = 8 * nt + 2 * (lane & 3);
                    const float2 sv = unpack2(sSb + r * GLDJ + c);
                    gc += ds[nt][2 * hf] * sv.x + ds[nt][2 * hf + 1] * sv.y;
                }
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) gc += __shfl_xor_sync(0xffffffffu, gc, o);
            if (lane == 0) spart[warp] = gc;
        }
        // dS <- gamma_{C-1} dS' + (diag(gamma) Q)^T dO (the part that does not wait for
        // dU); dU = diag(g) K dS' + P^T dO: 64 x 64, warp tile 16 x 32.  The three
        // products are independent and overlap in the MMA pipe.
        const float glast = sgb[64 + 63];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) ds[nt][e] *= glast;
        warp_mma_kscaled<8>(ds, sQ, LDT, sgb + 64, sO, GLDJ, 16 * warp, 0, C, lane);
        {
            const int m0 = 16 * (warp & 3), n0 = 32 * (warp >> 2);
            float du[4][4], pd[4][4];
            zero_acc(du);
            zero_acc(pd);
            warp_mma<0, 1, 4>(du, sK, LDT, sD, GLDJ, m0, n0, D, lane);
            warp_mma<1, 1, 4>(pd, sP, LDQ, sO, GLDJ, m0, n0, C, lane);
            bf16 *gdU = p.ws.dU + ch * 64 * D + j0;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const int r = m0 + (lane >> 2) + 8 * hf, c = n0 + 8 * nt + 2 * (lane & 3);
                    const float gr = sgb[128 + r];
                    const float a0 = gr * du[nt][2 * hf] + pd[nt][2 * hf];
                    const float a1 = gr * du[nt][2 * hf + 1] + pd[nt][2 * hf + 1];
                    *reinterpret_cast<uint32_t *>(gdU + (size_t)r * D + c) = pack2(a0, a1);
                    *reinterpret_cast<uint32_t *>(sdU + r * GLDJ + c) = pack2(-a0, -a1);
                }
        }
        __syncthreads();   // -dU and the partial sums complete
        if (tid == 0) {
            float t = 0.f;
            for (int w = 0; w < 8; ++w) t += spart[w];
            p.ws.gC[ch * kGcSlots + jb] = t;
        }
        // dS -= W^T dU: 128 x 64, K = 64
        warp_mma<1, 1, 8>(ds, sW, LDT, sdU, GLDJ, 16 * warp, 0, C, lane);
        __syncthreads();   // stage n and the dS', dO, dU tiles no longer read
        if (n >= 2) load(n - 2);
    }
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            const int r = 16 * warp + (lane >> 2) + 8 * hf, c = 8 * nt + 2 * (lane & 3);
            *reinterpret_cast<float2 *>(p.dS0 + hs + (size_t)r * D + j0 + c) =
                make_float2(ds[nt][2 * hf], ds[nt][2 * hf + 1]);
        }
}

// ================================================================== 4. chunk gradients
// Per (chunk n, QK head hq, sequence b), K3W = 16 warps.  Warp tiles: 64 x 128
// outputs 16 x 32 (rows 16 (w & 3), columns 32 (w >> 2)); 64 x 64 outputs 16 x 16.
// Row sums of a product come from the K3H = 4 warps of a row block, column sums of
// a 64 x 64 one from four: each writes its own slot ([4][64]) and the slots are
// added in a fixed order.
constexpr size_t K_Q = 0;
constexpr size_t K_K = K_Q + 64 * LDT * 2;
constexpr size_t K_V = K_K + 64 * LDT * 2;
constexpr size_t K_O = K_V + 64 * LDT * 2;      // dO
constexpr size_t K_U = K_O + 64 * LDT * 2;
constexpr size_t K_DU = K_U + 64 * LDT * 2;
constexpr size_t K_DW = K_DU + 64 * LDT * 2;    // dW = -dU S^T, bf16
constexpr size_t K_S = K_DW + 64 * LDT * 2;     // S, then dS' (128 x 128, [d][j])
constexpr size_t K_T = K_S + 128 * LDT * 2;
constexpr size_t K_X1 = K_T + 64 * LDQ * 2;     // dP o Gam, then Z = T^T dT
constexpr size_t K_X2 = K_X1 + 64 * LDQ * 2;    // dT, then M
constexpr size_t K_KK = K_X2 + 64 * LDQ * 2;
constexpr size_t K_QK = K_KK + 64 * LDF * 4;
constexpr size_t K_VEC = K_QK + 64 * LDF * 4;   // b, beta, gamma, g (64 each)
constexpr int NROW = 7;                         // row-sum arrays, [K3H][64] each
constexpr size_t K_ROW = K_VEC + 4 * 64 * 4;
constexpr size_t K_COL = K_ROW + NROW * K3H * 64 * 4;   // two column-sum arrays, [4][64] each
constexpr size_t K_BYTES = K_COL + 2 * 4 * 64 * 4;
enum { R_DGAM = 0, R_DBG, R_DB2, R_DG, R_GGP, R_GGA, R_DB3 };

constexpr int K3U = 4;                          // k-loop unroll of its MMAs (registers)

__global__ void __launch_bounds__(K3T, 1) grad_chunk_kernel(const Params p)
{
    extern __shared__ __align__(128) unsigned char smem[];
    bf16 *sQ = reinterpret_cast<bf16 *>(smem + K_Q), *sK = reinterpret_cast<bf16 *>(smem + K_K);
    bf16 *sV = reinterpret_cast<bf16 *>(smem + K_V), *sO = reinterpret_cast<bf16 *>(smem + K_O);
    bf16 *sU = reinterpret_cast<bf16 *>(smem + K_U), *sdU = reinterpret_cast<bf16 *>(smem + K_DU);
    bf16 *sdW = reinterpret_cast<bf16 *>(smem + K_DW), *sS = reinterpret_cast<bf16 *>(smem + K_S);
    bf16 *sT = reinterpret_cast<bf16 *>(smem + K_T);
    bf16 *sX1 = reinterpret_cast<bf16 *>(smem + K_X1), *sX2 = reinterpret_cast<bf16 *>(smem + K_X2);
    float *fKK = reinterpret_cast<float *>(smem + K_KK), *fQK = reinterpret_cast<float *>(smem + K_QK);
    float *vb = reinterpret_cast<float *>(smem + K_VEC), *vbeta = vb + 64, *vgam = vb + 128, *vg = vb + 192;
    float *rows = reinterpret_cast<float *>(smem + K_ROW);   // [NROW][K3H][64]
    float *cols = reinterpret_cast<float *>(smem + K_COL);   // [2][4][64]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n = blockIdx.x, hq = blockIdx.y, b = blockIdx.z;
    const int grp = p.Hv / p.Hqk;
    const int t0 = n * C, L = min(C, p.T - t0);
    const size_t qk_ld = (size_t)p.Hqk * D, v_ld = (size_t)p.Hv * D;
    const size_t tok = (size_t)b * p.T + t0;
    const int m0 = 16 * (warp & 3), n0 = 8 * NTA * (warp >> 2), n0p = 8 * NTB * (warp >> 2), wh = warp >> 2;
    const int g4 = lane >> 2, t4 = lane & 3;
    // a head's tiles: V, dO, U, dU, S (freed after dT is formed) and T (freed after dA)
    auto load_main = [&](int i) {
        const int h = hq * grp + i;
        const size_t ch = ((size_t)b * p.Hv + h) * p.NC + n;
        load_tile<64, 16, K3T>(sV, LDT, p.v + tok * v_ld + (size_t)h * D, v_ld, L, tid);
        load_tile<64, 16, K3T>(sO, LDT, p.dO + tok * v_ld + (size_t)h * D, v_ld, L, tid);
        load_tile<64, 16, K3T>(sU, LDT, p.ws.U + ch * 64 * D, D, 64, tid);
        load_tile<64, 16, K3T>(sdU, LDT, p.ws.dU + ch * 64 * D, D, 64, tid);
        load_tile<128, 16, K3T>(sS, LDT, p.ws.S + ch * D * D, D, 128, tid);
        cp_commit();
    };
    auto load_t = [&](int i) {
        const size_t ch = ((size_t)b * p.Hv + hq * grp + i) * p.NC + n;
        load_tile<64, 8, K3T>(sT, LDQ, p.ws.Tm + ch * 64 * 64, 64, 64, tid);
        cp_commit();
    };
    float nb = 0.f, nbeta = 0.f, ngam = 0.f, ng = 0.f;   // the next head's gates (tid < 64)
    auto fetch_gates = [&](int i) {
        if (tid < 64) {
            const int h = hq * grp + i;
            const float *gv = p.ws.gate + (((size_t)b * p.Hv + h) * p.NC + n) * 192;
            nb = gv[tid];
            nbeta = tid < L ? p.beta[(tok + tid) * p.Hv + h] : 0.f;
            ngam = gv[64 + tid];
            ng = gv[128 + tid];
        }
    };
    load_tile<64, 16, K3T>(sQ, LDT, p.q + tok * qk_ld + (size_t)hq * D, qk_ld, L, tid);
    load_tile<64, 16, K3T>(sK, LDT, p.k + tok * qk_ld + (size_t)hq * D, qk_ld, L, tid);
    cp_commit();
    load_main(0);
    load_t(0);
    fetch_gates(0);
    cp_wait<2>();
    __syncthreads();
    chunk_grams(sK, sQ, fKK, fQK, warp, lane);
    float dq[NTA][4], dk[NTA][4], x[NTA][4];
    zero_acc(dq);
    zero_acc(dk);
    // row partial of a 64 x 128 / 64 x 64 fragment: v[hf] for rows m0 + g4 + 8 hf
    auto put_rows = [&](int which, float v0, float v1) {
        v0 += __shfl_xor_sync(0xffffffffu, v0, 1);
        v0 += __shfl_xor_sync(0xffffffffu, v0, 2);
        v1 += __shfl_xor_sync(0xffffffffu, v1, 1);
        v1 += __shfl_xor_sync(0xffffffffu, v1, 2);
        if (t4 == 0) {
            rows[(which * K3H + wh) * 64 + m0 + g4] = v0;
            rows[(which * K3H + wh) * 64 + m0 + g4 + 8] = v1;
        }
    };
    auto row_sum = [&](int which, int r) {
        float t = 0.f;
#pragma unroll
        for (int q = 0; q < K3H; ++q) t += rows[(which * K3H + q) * 64 + r];
        return t;
    };
    for (int i = 0; i < grp; ++i) {
        const int h = hq * grp + i;
        const size_t ch = ((size_t)b * p.Hv + h) * p.NC + n;
        __syncthreads();   // grams written; the previous head's gates and sums no longer read
        if (tid < 64) {
            vb[tid] = nb;
            vbeta[tid] = nbeta;
            vgam[tid] = ngam;
            vg[tid] = ng;
        }
        cp_wait_all();
        __syncthreads();   // this head's tiles (loaded during the previous head) and gates
        // X1 = dO S^T: dQ += diag(gamma) X1; dgamma partial = rowsum(Q o X1)
        zero_acc(x);
        warp_mma<0, 0, NTA, K3U>(x, sO, LDT, sS, LDT, m0, n0, D, lane);
        {
            float r0 = 0.f, r1 = 0.f;
#pragma unroll
            for (int nt = 0; nt < NTA; ++nt)
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const int r = m0 + g4 + 8 * hf, c = n0 + 8 * nt + 2 * t4;
                    const float2 qv = unpack2(sQ + r * LDT + c);
                    const float ga = vgam[r];
                    dq[nt][2 * hf] += ga * x[nt][2 * hf];
                    dq[nt][2 * hf + 1] += ga * x[nt][2 * hf + 1];
                    const float t = qv.x * x[nt][2 * hf] + qv.y * x[nt][2 * hf + 1];
                    if (hf) r1 += t; else r0 += t;
                }
            put_rows(R_DGAM, r0, r1);
        }
        // X2 = dU S^T, dW = -X2 (bf16 tile)
        zero_acc(x);
        warp_mma<0, 0, NTA, K3U>(x, sdU, LDT, sS, LDT, m0, n0, D, lane);
#pragma unroll
        for (int nt = 0; nt < NTA; ++nt)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const int r = m0 + g4 + 8 * hf, c = n0 + 8 * nt + 2 * t4;
                *reinterpret_cast<uint32_t *>(sdW + r * LDT + c) = pack2(-x[nt][2 * hf], -x[nt][2 * hf + 1]);
            }
        __syncthreads();   // S no longer read; dW complete
        load_tile<128, 16, K3T>(sS, LDT, p.ws.dSp + ch * D * D, D, 128, tid);   // dS' (waited below)
        cp_commit();
        // dP = dO U^T (64 x 64); dP o Gam -> X1; Gam-weighted dP o QK row / column sums
        {
            float pp[NTB][4];
            zero_acc(pp);
            warp_mma<0, 0, NTB, K3U>(pp, sO, LDT, sU, LDT, m0, n0p, D, lane);
            float r0 = 0.f, r1 = 0.f, cs[NTB][2];
#pragma unroll
            for (int nt = 0; nt < NTB; ++nt) {
                cs[nt][0] = cs[nt][1] = 0.f;
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const int r = m0 + g4 + 8 * hf, c = n0p + 8 * nt + 2 * t4;
                    float o2[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int s = c + e;
                        const float gam = s <= r ? __expf(vb[r] - vb[s]) : 0.f;
                        const float dpg = pp[nt][2 * hf + e] * gam;
                        o2[e] = dpg;
                        const float gg = dpg * fQK[r * LDF + s];
                        if (hf) r1 += gg; else r0 += gg;
                        cs[nt][e] += gg;
                    }
                    *reinterpret_cast<uint32_t *>(sX1 + r * LDQ + c) = pack2(o2[0], o2[1]);
                }
            }
            put_rows(R_GGP, r0, r1);
#pragma unroll
            for (int nt = 0; nt < NTB; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    float v = cs[nt][e];
                    v += __shfl_xor_sync(0xffffffffu, v, 4);
                    v += __shfl_xor_sync(0xffffffffu, v, 8);
                    v += __shfl_xor_sync(0xffffffffu, v, 16);
                    if (g4 == 0) cols[(0 * 4 + (warp & 3)) * 64 + n0p + 8 * nt + 2 * t4 + e] = v;
                }
        }
        __syncthreads();   // X1 = dP o Gam complete
        warp_mma<0, 1, NTA, K3U>(dq, sX1, LDQ, sK, LDT, m0, n0, C, lane);   // dQ += (dP o Gam) K
        warp_mma<1, 1, NTA, K3U>(dk, sX1, LDQ, sQ, LDT, m0, n0, C, lane);   // dK += (dP o Gam)^T Q
        // T^T dW: dK += diag(beta gamma) T^T dW; dbg partial = rowsum(T^T dW o K)
        zero_acc(x);
        warp_mma<1, 1, NTA, K3U>(x, sT, LDQ, sdW, LDT, m0, n0, C, lane);
        {
            float r0 = 0.f, r1 = 0.f;
#pragma unroll
            for (int nt = 0; nt < NTA; ++nt)
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const int r = m0 + g4 + 8 * hf, c = n0 + 8 * nt + 2 * t4;
                    const float bg = vbeta[r] * vgam[r];
                    const float2 kv = unpack2(sK + r * LDT + c);
                    dk[nt][2 * hf] += bg * x[nt][2 * hf];
                    dk[nt][2 * hf + 1] += bg * x[nt][2 * hf + 1];
                    const float t = kv.x * x[nt][2 * hf] + kv.y * x[nt][2 * hf + 1];
                    if (hf) r1 += t; else r0 += t;
                }
            put_rows(R_DBG, r0, r1);
        }
        // T^T dU: dV = diag(beta) T^T dU; rowsum(T^T dU o V)
        zero_acc(x);
        warp_mma<1, 1, NTA, K3U>(x, sT, LDQ, sdU, LDT, m0, n0, C, lane);
        {
            float r0 = 0.f, r1 = 0.f;
#pragma unroll
            for (int nt = 0; nt < NTA; ++nt)
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const int r = m0 + g4 + 8 * hf, c = n0 + 8 * nt + 2 * t4;
                    const float2 vv = unpack2(sV + r * LDT + c);
                    const float t = vv.x * x[nt][2 * hf] + vv.y * x[nt][2 * hf + 1];
                    if (hf) r1 += t; else r0 += t;
                    if (r < L)
                        *reinterpret_cast<float2 *>(p.dv + ((tok + r) * p.Hv + h) * D + c) =
                            make_float2(vbeta[r] * x[nt][2 * hf], vbeta[r] * x[nt][2 * hf + 1]);
                }
            put_rows(R_DB2, r0, r1);
        }
        cp_wait_all();
        __syncthreads();   // dS' landed; X1 free
        // X3 = U dS'^T: dK += diag(g) X3; dg partial = rowsum(K o X3)
        zero_acc(x);
        warp_mma<0, 0, NTA, K3U>(x, sU, LDT, sS, LDT, m0, n0, D, lane);
        {
            float r0 = 0.f, r1 = 0.f;
#pragma unroll
            for (int nt = 0; nt < NTA; ++nt)
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const int r = m0 + g4 + 8 * hf, c = n0 + 8 * nt + 2 * t4;
                    const float2 kv = unpack2(sK + r * LDT + c);
                    dk[nt][2 * hf] += vg[r] * x[nt][2 * hf];
                    dk[nt][2 * hf + 1] += vg[r] * x[nt][2 * hf + 1];
                    const float t = kv.x * x[nt][2 * hf] + kv.y * x[nt][2 * hf + 1];
                    if (hf) r1 += t; else r0 += t;
                }
            put_rows(R_DG, r0, r1);
        }
        // dT[r][m] = beta_m gamma_m (dW K^T)[r][m] + beta_m (dU V^T)[r][m] -> X2
        {
            float y1[NTB][4], y2[NTB][4];
            zero_acc(y1);
            zero_acc(y2);
            warp_mma<0, 0, NTB, K3U>(y1, sdW, LDT, sK, LDT, m0, n0p, D, lane);
            warp_mma<0, 0, NTB, K3U>(y2, sdU, LDT, sV, LDT, m0, n0p, D, lane);
#pragma unroll
            for (int nt = 0; nt < NTB; ++nt)
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const int r = m0 + g4 + 8 * hf, c = n0p + 8 * nt + 2 * t4;
                    const float a0 = vbeta[c] * (vgam[c] * y1[nt][2 * hf] + y2[nt][2 * hf]);
                    const float a1 = vbeta[c + 1] * (vgam[c + 1] * y1[nt][2 * hf + 1] + y2[nt][2 * hf + 1]);
                    *reinterpret_cast<uint32_t *>(sX2 + r * LDQ + c) = pack2(a0, a1);
                }
        }
        __syncthreads();   // dT complete; V, dO, U, dU, dS' no longer read
        if (i + 1 < grp) load_main(i + 1);
        // Z = T^T dT -> X1
        {
            float z[NTB][4];
            zero_acc(z);
            warp_mma<1, 1, NTB, K3U>(z, sT, LDQ, sX2, LDQ, m0, n0p, C, lane);
#pragma unroll
            for (int nt = 0; nt < NTB; ++nt)
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const int r = m0 + g4 + 8 * hf, c = n0p + 8 * nt + 2 * t4;
                    *reinterpret_cast<uint32_t *>(sX1 + r * LDQ + c) = pack2(z[nt][2 * hf], z[nt][2 * hf + 1]);
                }
        }
        __syncthreads();   // Z complete; dT no longer read
        // dA = -Z T^T (strictly lower): dbeta term rowsum(dA o Gam o KK), Gam-weighted
        // dA o beta KK row / column sums, M = diag(beta) (dA o Gam) -> X2
        {
            float a[NTB][4];
            zero_acc(a);
            warp_mma<0, 0, NTB, K3U>(a, sX1, LDQ, sT, LDQ, m0, n0p, C, lane);
            float r0 = 0.f, r1 = 0.f, q0 = 0.f, q1 = 0.f, cs[NTB][2];
#pragma unroll
            for (int nt = 0; nt < NTB; ++nt) {
                cs[nt][0] = cs[nt][1] = 0.f;
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const int r = m0 + g4 + 8 * hf, c = n0p + 8 * nt + 2 * t4;
                    float mm[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int s = c + e;
                        float t3 = 0.f, gg = 0.f, mv = 0.f;
                        if (s < r) {
                            const float da = -a[nt][2 * hf + e];
                            const float gam = __expf(vb[r] - vb[s]);
                            const float dgk = da * gam * fKK[r * LDF + s];
                            t3 = dgk;
                            gg = vbeta[r] * dgk;
                            mv = vbeta[r] * da * gam;
                        }
                        mm[e] = mv;
                        if (hf) { r1 += t3; q1 += gg; } else { r0 += t3; q0 += gg; }
                        cs[nt][e] += gg;
                    }
                    *reinterpret_cast<uint32_t *>(sX2 + r * LDQ + c) = pack2(mm[0], mm[1]);
                }
            }
            put_rows(R_DB3, r0, r1);
            put_rows(R_GGA, q0, q1);
#pragma unroll
            for (int nt = 0; nt < NTB; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    float v = cs[nt][e];
                    v += __shfl_xor_sync(0xffffffffu, v, 4);
                    v += __shfl_xor_sync(0xffffffffu, v, 8);
                    v += __shfl_xor_sync(0xffffffffu, v, 16);
                    if (g4 == 0) cols[(1 * 4 + (warp & 3)) * 64 + n0p + 8 * nt + 2 * t4 + e] = v;
                }
        }
        __syncthreads();   // M complete; every row / column sum written; T no longer read
        if (i + 1 < grp) {
            load_t(i + 1);
            fetch_gates(i + 1);
        }
        warp_mma<0, 1, NTA, K3U>(dk, sX2, LDQ, sK, LDT, m0, n0, C, lane);   // dK += M K
        warp_mma<1, 1, NTA, K3U>(dk, sX2, LDQ, sK, LDT, m0, n0, C, lane);   // dK += M^T K
        // gate gradients (warp 0, two rows per lane), then d log alpha by a reverse scan
        if (warp == 0) {
            float gc = 0.f;
#pragma unroll
            for (int q = 0; q < kGcSlots; ++q) gc += p.ws.gC[ch * kGcSlots + q];
            float db[2], dbeta_v[2], gsum = 0.f;
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int r = 2 * lane + e;
                const float dbg = row_sum(R_DBG, r);
                const float dgamma = row_sum(R_DGAM, r) + dbg * vbeta[r];
                dbeta_v[e] = dbg * vgam[r] + row_sum(R_DB2, r) + row_sum(R_DB3, r);
                float colsum = 0.f;
#pragma unroll
                for (int q = 0; q < 4; ++q) colsum += cols[(0 * 4 + q) * 64 + r] + cols[(1 * 4 + q) * 64 + r];
                const float gg = row_sum(R_DG, r) * vg[r];
                db[e] = dgamma * vgam[r] + row_sum(R_GGP, r) + row_sum(R_GGA, r) - colsum - gg;
                gsum += gg;
            }
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) gsum += __shfl_xor_sync(0xffffffffu, gsum, o);
            if (lane == 31) db[1] += gc * vgam[63] + gsum;
            // reverse inclusive scan: dla[r] = sum_{r' >= r} db[r']
            float s = db[0] + db[1];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_down_sync(0xffffffffu, s, o);
                if (lane + o < 32) s += y;
            }
            const float dla1 = s - db[0], dla0 = s;
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int r = 2 * lane + e;
                if (r < L) {
                    const size_t gi = (tok + r) * p.Hv + h;
                    p.dalpha[gi] = (e ? dla1 : dla0) / p.alpha[gi];
                    p.dbeta[gi] = dbeta_v[e];
                }
            }
        }
    }
    // dq, dk rows of this chunk (every V head of the group summed)
#pragma unroll
    for (int nt = 0; nt < NTA; ++nt)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            const int r = m0 + g4 + 8 * hf, c = n0 + 8 * nt + 2 * t4;
            if (r < L) {
                const size_t gi = ((tok + r) * p.Hqk + hq) * D + c;
                *reinterpret_cast<float2 *>(p.dq + gi) = make_float2(dq[nt][2 * hf], dq[nt][2 * hf + 1]);
                *reinterpret_cast<float2 *>(p.dk + gi) = make_float2(dk[nt][2 * hf], dk[nt][2 * hf + 1]);
            }
        }
}

// Workspace layout: the arrays of Ws in order, each 256-byte aligned.
struct WsLayout {
    size_t W, U, Tm, P, S, dSp, dU, gate, gC, bytes;
};
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
WsLayout ws_layout(int B, int T, int Hv)
{
    const size_t nch = (size_t)B * Hv * ((T + C - 1) / C);
    WsLayout l{};
    size_t o = 0;
    auto take = [&](size_t bytes) { const size_t at = o; o = align256(o + bytes); return at; };
    l.W = take(nch * 64 * D * 2);
    l.U = take(nch * 64 * D * 2);
    l.Tm = take(nch * 64 * 64 * 2);
    l.P = take(nch * 64 * 64 * 2);
    l.S = take(nch * D * D * 2);
    l.dSp = take(nch * D * D * 2);
    l.dU = take(nch * 64 * D * 2);
    l.gate = take(nch * 192 * 4);
    l.gC = take(nch * kGcSlots * 4);
    l.bytes = o;
    return l;
}

}  // namespace

size_t bwd_chunk_workspace(int B, int T, int Hv)
{
    if (B <= 0 || T <= 0) return 0;
    return ws_layout(B, T, Hv).bytes;
}

cudaError_t launch_bwd_chunk(const BwdLaunch &L, cudaStream_t stream)
{
    const size_t hs = (size_t)kHeadDim * kHeadDim;
    if (L.T == 0) {   // no tokens: dS0 = dS_final (zeros without it)
        const size_t bytes = (size_t)L.B * L.Hv * hs * sizeof(float);
        return L.dS_final ? cudaMemcpyAsync(L.dS0, L.dS_final, bytes, cudaMemcpyDeviceToDevice, stream)
                          : cudaMemsetAsync(L.dS0, 0, bytes, stream);
    }
    const WsLayout l = ws_layout(L.B, L.T, L.Hv);
    unsigned char *w = reinterpret_cast<unsigned char *>(L.work);
    Params p{};
    p.q = static_cast<const bf16 *>(L.q);
    p.k = static_cast<const bf16 *>(L.k);
    p.v = static_cast<const bf16 *>(L.v);
    p.dO = static_cast<const bf16 *>(L.dO);
    p.alpha = L.alpha;
    p.beta = L.beta;
    p.S0 = L.S0;
    p.dS_final = L.dS_final;
    p.dq = L.dq;
    p.dk = L.dk;
    p.dv = L.dv;
    p.dalpha = L.dalpha;
    p.dbeta = L.dbeta;
    p.dS0 = L.dS0;
    p.ws = Ws{reinterpret_cast<bf16 *>(w + l.W), reinterpret_cast<bf16 *>(w + l.U),
              reinterpret_cast<bf16 *>(w + l.Tm), reinterpret_cast<bf16 *>(w + l.P),
              reinterpret_cast<bf16 *>(w + l.S), reinterpret_cast<bf16 *>(w + l.dSp),
              reinterpret_cast<bf16 *>(w + l.dU), reinterpret_cast<float *>(w + l.gate),
              reinterpret_cast<float *>(w + l.gC)};
    p.B = L.B;
    p.T = L.T;
    p.Hqk = L.Hqk;
    p.Hv = L.Hv;
    p.NC = (L.T + C - 1) / C;
    cudaError_t err;
    if ((err = cudaFuncSetAttribute(prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)P_BYTES)))
        return err;
    if ((err = cudaFuncSetAttribute(fwd_chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)F_BYTES)))
        return err;
    if ((err = cudaFuncSetAttribute(grad_chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)G_BYTES)))
        return err;
    if ((err = cudaFuncSetAttribute(grad_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)K_BYTES)))
        return err;
    const dim3 per_chunk((unsigned)p.NC, (unsigned)L.Hqk, (unsigned)L.B);
    prep_kernel<<<per_chunk, kThreads, P_BYTES, stream>>>(p);
    fwd_chain_kernel<<<dim3((unsigned)(D / FJ), (unsigned)L.Hv, (unsigned)L.B), kThreads, F_BYTES, stream>>>(p);
    grad_chain_kernel<<<dim3((unsigned)(D / GJ), (unsigned)L.Hv, (unsigned)L.B), kThreads, G_BYTES, stream>>>(p);
    grad_chunk_kernel<<<per_chunk, K3T, K_BYTES, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace gdn
