// Chunkwise (WY) prefill on the 5th-generation tensor cores (tcgen05), bf16
// inputs, fp32 accumulation, fp32 state kept in tensor memory (TMEM).
//
// Source: "Qwen3.8-Flash-Next 技术总结 -- Qwen4 架构的探路者", section 2.1 "Gated
// DeltaNet": S_t = alpha_t S_{t-1} + beta_t k_t (v_t - alpha_t S_{t-1}^T k_t)^T,
// evaluated chunk by chunk with the WY representation.  Per chunk of C = 64
// tokens from state S (dk x dv), with b_r = sum_{j<=r} log alpha_j,
// gamma_r = exp(b_r), Gam[r,i] = exp(b_r - b_i) (i <= r), g_i = exp(b_{C-1} - b_i):
//   A      = strict_lower(beta_r Gam[r,i] k_r . k_i),   T = (I + A)^-1
//   W      = T diag(beta gamma) K,   U~ = T diag(beta) V
//   U      = U~ - W S
//   O      = diag(gamma) Q S + (Gam o Q K^T) U              (i <= r)
//   S     <- gamma_{C-1} S + (diag(g) K)^T U
//
// Every product is computed transposed so that its M dimension is a head
// dimension (128, the TMEM lanes: the tensor core's full-rate shape) and the 64
// chunk positions are N:
//   G    = [K;Q] K^T      (lanes 0-63: K K^T, lanes 64-127: Q K^T)    M=128 N=64  K=128
//   W^T  = K^T (T diag(beta gamma))^T                                  M=128 N=64  K=64
//   U^T  = V^T (T diag(beta))^T  -  S^T W^T                            M=128 N=64  K=64+128
//   O^T  = diag(gamma) (S^T Q^T) + U^T P^T,  P = masked Gam o Q K^T
//   S^T <- gamma_{C-1} S^T + U^T K~,  K~ = diag(g) K                   M=128 N=128 K=64
// The state S^T (128 lanes x 128 fp32 columns) stays in TMEM for the whole
// sequence; its bf16 copy in shared memory is only an MMA operand.
//
// One CTA per (sequence, V head), warp-specialised:
//   warp 0      TMA producer: K, Q (double-buffered) and V tiles, 128B swizzle
//   warp 1      MMA issuer (one thread), event-driven: it issues whichever MMA
//               group has its inputs ready, state-dependent groups first
//   warps 2-5   "prep" warpgroup, runs ahead of the state: gates, A and P from
//               the grams, the triangular solve (fp32 CUDA cores + TF32 warp
//               MMAs for the block merges), W^T to shared memory and K~
//   warps 6-9   "chain" warpgroup, the state-dependent path: S^T -> bf16
//               operand (+ decay of the fp32 state), U^T -> bf16 operand, the
//               gamma scaling of the S-part of O^T in TMEM, and the O epilogue
//               (staged in shared memory, one TMA store)
// The U^T and O^T accumulators are double-buffered, so the prep work of the
// next chunk never waits for the state-dependent chain of the current one.
//
// Every wait is bounded.  On a timeout the CTA raises a device error flag, the
// other roles see a shared abort flag and stop, in-flight copies and MMAs are
// drained (again with a bound) and TMEM is freed before returning.
#include <cuda.h>

#include "gdn_internal.cuh"
#include "sm100.cuh"

namespace gdn {

__device__ unsigned int g_tc_error = 0;   // set when a bounded wait gave up

// Optional event trace (build with -DGDN_TRACE): block (0, 0) records %globaltimer
// at fixed points of every role for the first kTraceChunks chunks.
#ifdef GDN_TRACE
constexpr int kTraceChunks = 16, kTraceSlots = 32;
__device__ unsigned long long g_trace[kTraceChunks][kTraceSlots];
__device__ __forceinline__ void trace(int c, int slot, bool leader) {
    if (leader && blockIdx.x == 0 && blockIdx.y == 0 && c < kTraceChunks) {
        unsigned long long t;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        g_trace[c][slot] = t;
    }
}
#define GDN_TRACE_AT(c, slot, leader) trace((c), (slot), (leader))
#else
#define GDN_TRACE_AT(c, slot, leader) ((void)0)
#endif

namespace {

using namespace sm100;

constexpr int C = kChunk;          // 64
constexpr int NT = 320;            // 10 warps
constexpr uint32_t TILE = 8192;    // one 64 x 64 bf16 tile, 128B-swizzled

// TMEM columns (fp32 accumulators over 128 lanes)
constexpr uint32_t COL_S = 0;      // S^T: 128 columns
constexpr uint32_t COL_G = 128;    // [K;Q] K^T
constexpr uint32_t COL_W = 192;    // W^T
constexpr uint32_t COL_U = 256;    // U^T, two buffers (256, 320)
constexpr uint32_t COL_O = 384;    // O^T, two buffers (384, 448)
constexpr uint32_t TMEM_COLS = 512;

// Shared-memory plan (byte offsets from a 1024-aligned base).
constexpr uint32_t OFF_KQ = 0;                    // 2 stages x [K d0-63][Q d0-63][K d64-127][Q d64-127]
constexpr uint32_t KQ_STAGE = 4 * TILE;
constexpr uint32_t OFF_V = OFF_KQ + 2 * KQ_STAGE; // [V j0-63][V j64-127]
constexpr uint32_t OFF_KT = OFF_V + 2 * TILE;     // K~ = diag(g) K, same layout as [K0][K1]
constexpr uint32_t OFF_P = OFF_KT + 2 * TILE;     // 2 x P [r][i] K-major
constexpr uint32_t OFF_BW = OFF_P + 2 * TILE;     // T diag(beta gamma) [r][i]
constexpr uint32_t OFF_BU = OFF_BW + TILE;        // T diag(beta)       [r][i]
constexpr uint32_t OFF_W = OFF_BU + TILE;         // W stored [d][r] (MN-major B), 128 rows
constexpr uint32_t OFF_S = OFF_W + 2 * TILE;      // S^T bf16 [j][d], two 64-column halves
constexpr uint32_t OFF_U = OFF_S + 4 * TILE;      // U^T bf16 [j][i]; between chunks: O staging [r][j]
constexpr uint32_t OFF_A = OFF_U + 2 * TILE;      // A, then T = (I + A)^-1, fp32 [64][LDA]
constexpr int LDA = 68;                           // padded row stride (floats)
constexpr uint32_t OFF_Y = OFF_A + 64 * LDA * 4;  // solve scratch, fp32 [32][LDY]
constexpr int LDY = 40;
// per-chunk gate vectors (2 buffers): b (log2 units), gamma, beta, g, beta*gamma,
// alpha (as used: 2^(clamped log2 alpha)), and d31[i] = prod_{i<j<=31} alpha_j (i < 32)
constexpr uint32_t OFF_GATE = OFF_Y + 32 * LDY * 4;
constexpr int GV_B = 0, GV_GAM = 64, GV_BETA = 128, GV_G = 192, GV_BG = 256, GV_ALPHA = 320,
              GV_D31 = 384;
constexpr uint32_t GATE_BUF = 416 * 4;
constexpr uint32_t OFF_BAR = OFF_GATE + 2 * GATE_BUF;
constexpr uint32_t NBAR = 23;
constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;    // tmem slot, abort flag
constexpr uint32_t SMEM_USED = OFF_MISC + 16;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;    // slack for aligning the base

// barrier indices (arrival count 1 unless noted)
enum : int {
    B_KQ_FULL = 0,   // 2: TMA K/Q stage landed
    B_KQ_EMPTY = 2,  // 2: stage no longer read
    B_V_FULL = 4, B_V_EMPTY = 5,
    B_G_FULL = 6,    // grams done
    B_W_FULL = 7,    // W^T, U~^T done
    B_SOLVE = 8,     // prep: Bw, Bu, P written (128)
    B_PREP = 9,      // prep: W, K~ written (128)
    B_GATES = 10,    // 2: gates of a chunk written
    B_S_READY = 12,  // chain: S^T bf16 written (128)
    B_U_FULL = 13,   // U^T done
    B_U_READY = 14,  // chain: U^T bf16 of a chunk with even index written (128); odd: B_U_READY1
    B_S_FULL = 15,   // state update done
    B_O_FREE = 16,   // 2: O accumulator read out (128)
    B_DRAIN = 18,    // final MMA drain
    B_G_FREE = 19,   // prep: grams read out of TMEM (128)
    B_U_READY1 = 20,
    B_X_FULL = 21,   // S-part of O^T (S^T Q^T) done
    B_O_FULL = 22,   // O^T complete (after U^T P^T)
};
// One U_READY barrier per U^T buffer, so that a parity probe of chunk c - 2's
// phase can never alias with a later completion on the same barrier.
__host__ __device__ constexpr int u_ready(int c) { return (c & 1) ? B_U_READY1 : B_U_READY; }

constexpr uint32_t ID_G = idesc_bf16(128, 64, false, false);
constexpr uint32_t ID_W = idesc_bf16(128, 64, true, false);
constexpr uint32_t ID_UT = idesc_bf16(128, 64, true, false);
constexpr uint32_t ID_U = idesc_bf16(128, 64, false, true, /*neg_b=*/true);
constexpr uint32_t ID_O = idesc_bf16(128, 64, false, false);
constexpr uint32_t ID_S = idesc_bf16(128, 128, false, true);

constexpr float kLog2Floor = -87.0f * 1.4426950408889634f;   // log alpha >= -87

struct TcParams {
    const float *alpha, *beta, *S0;
    float *S_final;
    int T, Hqk, Hv;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// 64 fp32 values (one row) -> bf16 row `row` of a 128B-swizzled tile.
__device__ __forceinline__ void store_row_bf16(unsigned char *tile, uint32_t row, const float *x) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        uint4 v;
        v.x = pack_bf16x2(x[8 * c + 0], x[8 * c + 1]);
        v.y = pack_bf16x2(x[8 * c + 2], x[8 * c + 3]);
        v.z = pack_bf16x2(x[8 * c + 4], x[8 * c + 5]);
        v.w = pack_bf16x2(x[8 * c + 6], x[8 * c + 7]);
        *reinterpret_cast<uint4 *>(tile + sw128_chunk(row, c)) = v;
    }
}

// 32 fp32 values -> bf16 elements 32*half .. 32*half+31 of row `row` (4 chunks).
__device__ __forceinline__ void store_half_row_bf16(unsigned char *tile, uint32_t row, int half,
                                                    const float *x) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint4 v;
        v.x = pack_bf16x2(x[8 * c + 0], x[8 * c + 1]);
        v.y = pack_bf16x2(x[8 * c + 2], x[8 * c + 3]);
        v.z = pack_bf16x2(x[8 * c + 4], x[8 * c + 5]);
        v.w = pack_bf16x2(x[8 * c + 6], x[8 * c + 7]);
        *reinterpret_cast<uint4 *>(tile + sw128_chunk(row, 4 * half + c)) = v;
    }
}

// Scales row `row` (64 bf16, swizzled) of a tile in place / into another tile.
__device__ __forceinline__ void scale_row_bf16(const unsigned char *src, unsigned char *dst,
                                               uint32_t row, float s) {
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
        const uint32_t off = sw128_chunk(row, ch);
        uint4 v = *reinterpret_cast<const uint4 *>(src + off);
        __nv_bfloat162 *hv = reinterpret_cast<__nv_bfloat162 *>(&v);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(hv[e]);
            hv[e] = __floats2bfloat162_rn(f.x * s, f.y * s);
        }
        *reinterpret_cast<uint4 *>(dst + off) = v;
    }
}

__device__ __forceinline__ void named_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// Named barrier that also returns the AND of `v` over the participating threads.
__device__ __forceinline__ bool named_and(int id, int nthreads, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.and.pred p, %2, %3, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r) : "r"((uint32_t)v), "r"(id), "r"(nthreads) : "memory");
    return r != 0;
}
// Non-blocking probe of an mbarrier phase.
__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return done != 0;
}

// ---------------------------------------------------------------- triangular solve
// T = (I + A)^-1 for the 64 x 64 strictly lower A in sA (row stride LDA), in place,
// by the 128 threads of one warpgroup (named barrier `bid`).  Blocked: 8 x 8
// diagonal blocks by substitution, then merges 8 -> 16 on CUDA cores and
// 16 -> 32 -> 64 with warp-level TF32 tensor-core products, using
// T_ba = -T_bb (A_ba T_aa) for the block below the diagonal of each merge.
// (The merges are 16- and 32-wide products: too small for a tcgen05 tile and
// its TMEM round trip, so they run as register-resident warp MMAs.)
__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
// d (16 x 8 fp32 fragment) += X[xr0.., xc0..xc0+8) * Y[yr0..yr0+8, yc0..yc0+8)
__device__ __forceinline__ void mma_tf32_step(float *d, const float *X, int ldx, int xr0, int xc0,
                                              const float *Y, int ldy, int yr0, int yc0, int lane) {
    const int g = lane >> 2, t = lane & 3;
    const uint32_t a0 = to_tf32(X[(xr0 + g) * ldx + xc0 + t]);
    const uint32_t a1 = to_tf32(X[(xr0 + g + 8) * ldx + xc0 + t]);
    const uint32_t a2 = to_tf32(X[(xr0 + g) * ldx + xc0 + t + 4]);
    const uint32_t a3 = to_tf32(X[(xr0 + g + 8) * ldx + xc0 + t + 4]);
    const uint32_t b0 = to_tf32(Y[(yr0 + t) * ldy + yc0 + g]);
    const uint32_t b1 = to_tf32(Y[(yr0 + t + 4) * ldy + yc0 + g]);
    asm(   // not volatile: lets the compiler hoist the fragment loads of later steps
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void store_frag(float *D, int ldd, int r0, int c0, const float *d,
                                           float s, int lane) {
    const int g = lane >> 2, t = lane & 3;
    D[(r0 + g) * ldd + c0 + 2 * t] = s * d[0];
    D[(r0 + g) * ldd + c0 + 2 * t + 1] = s * d[1];
    D[(r0 + g + 8) * ldd + c0 + 2 * t] = s * d[2];
    D[(r0 + g + 8) * ldd + c0 + 2 * t + 1] = s * d[3];
}

__device__ void unit_lower_inverse(float *sA, float *sY, int t, int bid) {
    const int warp = t >> 5, lane = t & 31;
    // 8 x 8 diagonal blocks: thread (block kb, column cl), right-looking substitution
    if (t < 64) {
        const int kb = t >> 3, cl = t & 7;
        float x[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) x[r] = (r == cl) ? 1.f : 0.f;
#pragma unroll
        for (int r = 0; r < 7; ++r) {
            const float xr = x[r];
#pragma unroll
            for (int q = r + 1; q < 8; ++q) x[q] = fmaf(-sA[(8 * kb + q) * LDA + 8 * kb + r], xr, x[q]);
        }
        named_sync(bid, 128);
#pragma unroll
        for (int r = 0; r < 8; ++r) sA[(8 * kb + r) * LDA + 8 * kb + cl] = x[r];
    } else {
        named_sync(bid, 128);
    }
    named_sync(bid, 128);
    // 8 -> 16 inside each 16 x 16 diagonal block: thread (block k, row r, 2 columns)
    {
        const int k = t >> 5, r = (t >> 2) & 7, c0 = (t & 3) * 2;
        const int ra = 16 * k, rb = 16 * k + 8;
        float y0 = 0.f, y1 = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float av = sA[(rb + r) * LDA + ra + i];
            y0 = fmaf(av, sA[(ra + i) * LDA + ra + c0], y0);
            y1 = fmaf(av, sA[(ra + i) * LDA + ra + c0 + 1], y1);
        }
        sY[k * 64 + r * 8 + c0] = y0;
        sY[k * 64 + r * 8 + c0 + 1] = y1;
        named_sync(bid, 128);
        float z0 = 0.f, z1 = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float tv = sA[(rb + r) * LDA + rb + i];
            z0 = fmaf(-tv, sY[k * 64 + i * 8 + c0], z0);
            z1 = fmaf(-tv, sY[k * 64 + i * 8 + c0 + 1], z1);
        }
        sA[(rb + r) * LDA + ra + c0] = z0;
        sA[(rb + r) * LDA + ra + c0 + 1] = z1;
    }
    named_sync(bid, 128);
    // 16 -> 32 for the blocks (16-31, 0-15) and (48-63, 32-47): warp -> (block, 8-column tile)
    {
        const int blk = warp >> 1, nt = warp & 1;
        const int a = 32 * blk, bb = a + 16;
        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < 2; ++ks)
            mma_tf32_step(d, sA, LDA, bb, a + 8 * ks, sA, LDA, a + 8 * ks, a + 8 * nt, lane);
        store_frag(sY + blk * 16 * LDY, LDY, 0, 8 * nt, d, 1.f, lane);
        named_sync(bid, 128);
        float e[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < 2; ++ks)
            mma_tf32_step(e, sA, LDA, bb, bb + 8 * ks, sY + blk * 16 * LDY, LDY, 8 * ks, 8 * nt, lane);
        store_frag(sA, LDA, bb, a + 8 * nt, e, -1.f, lane);
    }
    named_sync(bid, 128);
    // 32 -> 64 for the block (32-63, 0-31): warp -> (16-row tile, two 8-column tiles)
    {
        const int mt = warp >> 1, n0 = 2 * (warp & 1);
        float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            mma_tf32_step(d0, sA, LDA, 32 + 16 * mt, 8 * ks, sA, LDA, 8 * ks, 8 * n0, lane);
            mma_tf32_step(d1, sA, LDA, 32 + 16 * mt, 8 * ks, sA, LDA, 8 * ks, 8 * (n0 + 1), lane);
        }
        store_frag(sY, LDY, 16 * mt, 8 * n0, d0, 1.f, lane);
        store_frag(sY, LDY, 16 * mt, 8 * (n0 + 1), d1, 1.f, lane);
        named_sync(bid, 128);
        float e0[4] = {0.f, 0.f, 0.f, 0.f}, e1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            mma_tf32_step(e0, sA, LDA, 32 + 16 * mt, 32 + 8 * ks, sY, LDY, 8 * ks, 8 * n0, lane);
            mma_tf32_step(e1, sA, LDA, 32 + 16 * mt, 32 + 8 * ks, sY, LDY, 8 * ks, 8 * (n0 + 1), lane);
        }
        store_frag(sA, LDA, 32 + 16 * mt, 8 * n0, e0, -1.f, lane);
        store_frag(sA, LDA, 32 + 16 * mt, 8 * (n0 + 1), e1, -1.f, lane);
    }
    named_sync(bid, 128);
}

// alpha, beta of tokens 2*lane, 2*lane+1 of chunk cn (alpha = 1, beta = 0 past the end)
__device__ __forceinline__ void load_gates(const TcParams &p, int b, int h, int T, int cn, int lane,
                                           float &a0, float &a1, float &b0, float &b1) {
    const int tn = cn * C, Ln = min(C, T - tn);
    const int r = 2 * lane;
    const size_t gi = ((size_t)b * T + tn + r) * p.Hv + h;
    a0 = r < Ln ? p.alpha[gi] : 1.f;
    b0 = r < Ln ? p.beta[gi] : 0.f;
    a1 = r + 1 < Ln ? p.alpha[gi + p.Hv] : 1.f;
    b1 = r + 1 < Ln ? p.beta[gi + p.Hv] : 0.f;
}

struct Ctl {
    uint64_t *bar;
    volatile int *abort_flag;
    // Bounded wait that also gives up as soon as another role aborted.  The
    // thread sleeps in the barrier unit between checks, so waiting roles do not
    // take issue slots from the working ones.
    __device__ __forceinline__ bool wait(int i, uint32_t parity) const {
        if (mbar_try_wait(&bar[i], parity)) return true;
        const long long t0 = clock64();
        for (;;) {
            if (mbar_try_wait_suspend(&bar[i], parity, 20000)) return true;
            if (*abort_flag) return false;
            if (clock64() - t0 > (1ll << 32)) {
                *abort_flag = 1;
                atomicOr(&g_tc_error, 1u);
                return false;
            }
        }
    }
};

__global__ void __launch_bounds__(NT, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                const TcParams p)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // Align by offsetting the shared array itself (not via an integer round trip), so
    // the compiler keeps every access below in the shared state space (LDS/STS).
    unsigned char *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + OFF_MISC + 4);
    const Ctl ctl{bar, abort_flag};

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.x, b = blockIdx.y;
    const int hq = h / (p.Hv / p.Hqk);
    const int T = p.T;
    const int nchunks = (T + C - 1) / C;
    const uint32_t sbase = smem_u32(sm);

    if (tid == 0) {
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_v);
        prefetch_tensormap(&tm_o);
        for (int i = 0; i < (int)NBAR; ++i) {
            const bool many = (i == B_SOLVE || i == B_PREP || i == B_S_READY || i == B_U_READY ||
                               i == B_U_READY1 || i == B_O_FREE || i == B_O_FREE + 1 ||
                               i == B_G_FREE);
            mbar_init(&bar[i], many ? 128 : 1);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ======================================================== TMA producer
        if (lane == 0) {
            bool ok = true;
            int issued_kq0 = -1, issued_kq1 = -1, issued_v = -1;
            for (int c = 0; c < nchunks && ok; ++c) {
                const int s = c & 1, t0 = c * C;
                if (c >= 2) ok = ctl.wait(B_KQ_EMPTY + s, ((c >> 1) - 1) & 1);
                if (!ok) break;
                unsigned char *st = sm + OFF_KQ + s * KQ_STAGE;
                mbar_arrive_expect_tx(&bar[B_KQ_FULL + s], KQ_STAGE);
                tma_load_4d(st + 0 * TILE, &tm_k, &bar[B_KQ_FULL + s], 0, hq, t0, b);
                tma_load_4d(st + 1 * TILE, &tm_q, &bar[B_KQ_FULL + s], 0, hq, t0, b);
                tma_load_4d(st + 2 * TILE, &tm_k, &bar[B_KQ_FULL + s], 64, hq, t0, b);
                tma_load_4d(st + 3 * TILE, &tm_q, &bar[B_KQ_FULL + s], 64, hq, t0, b);
                if (s) issued_kq1 = c; else issued_kq0 = c;
                if (c >= 1) ok = ctl.wait(B_V_EMPTY, (c - 1) & 1);
                if (!ok) break;
                mbar_arrive_expect_tx(&bar[B_V_FULL], 2 * TILE);
                tma_load_4d(sm + OFF_V, &tm_v, &bar[B_V_FULL], 0, h, t0, b);
                tma_load_4d(sm + OFF_V + TILE, &tm_v, &bar[B_V_FULL], 64, h, t0, b);
                issued_v = c;
            }
            if (*abort_flag) {
                // Let copies still in flight land before the CTA's memory goes away.
                if (issued_kq0 >= 0) mbar_wait(&bar[B_KQ_FULL], (issued_kq0 >> 1) & 1, 1ll << 28);
                if (issued_kq1 >= 0) mbar_wait(&bar[B_KQ_FULL + 1], (issued_kq1 >> 1) & 1, 1ll << 28);
                if (issued_v >= 0) mbar_wait(&bar[B_V_FULL], issued_v & 1, 1ll << 28);
            }
        }
    } else if (warp == 1) {
        // ======================================================== MMA issuer
        // Issues, as soon as their inputs are ready, in this priority order:
        //   YS(c): O^T += U^T P^T, S^T += U^T K~     needs U^T bf16 of chunk c
        //   UO(c): U^T += S^T (-W)^T, O^T = S^T Q^T   needs S^T bf16 and prep of c
        //   WU(c): W^T, U~^T                          needs the solve of c
        //   G(c):  [K;Q] K^T                          needs the K/Q tiles of c
        if (lane == 0) {
            int ng = 0, nwu = 0, nuo = 0, nys = 0;
            long long idle_since = clock64();
            while (nys < nchunks) {
                if (*abort_flag) break;
                bool issued = false;
                if (nys < nuo && mbar_test(&bar[u_ready(nys)], (nys >> 1) & 1)) {
                    const int c = nys, s = c & 1;
                    tc_fence_after();
                    const uint32_t col_o = COL_O + s * 64;
                    // the state update first: the next chunk waits for it
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_bf16(tmem + COL_S, smem_desc_sw128(sbase + OFF_U + k * 32, 16, 1024),
                                 smem_desc_sw128(sbase + OFF_KT + k * 2048, TILE, 1024), ID_S, true);
                    mma_commit(&bar[B_S_FULL]);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_bf16(tmem + col_o, smem_desc_sw128(sbase + OFF_U + k * 32, 16, 1024),
                                 smem_desc_sw128(sbase + OFF_P + s * TILE + k * 32, 16, 1024), ID_O, true);
                    mma_commit(&bar[B_O_FULL]);
                    GDN_TRACE_AT(c, 5, true);
                    ++nys;
                    issued = true;
                } else if (nuo < nwu && mbar_test(&bar[B_PREP], nuo & 1) &&
                           mbar_test(&bar[B_S_READY], nuo & 1) &&
                           (nuo < 2 || mbar_test(&bar[B_O_FREE + (nuo & 1)], ((nuo >> 1) - 1) & 1))) {
                    const int c = nuo, s = c & 1;
                    const uint32_t st = sbase + OFF_KQ + s * KQ_STAGE;
                    const uint32_t col_o = COL_O + s * 64, col_u = COL_U + s * 64;
                    tc_fence_after();
                    GDN_TRACE_AT(c, 1, true);
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint32_t koff = (k >> 2) * 2 * TILE + (k & 3) * 32;
                        mma_bf16(tmem + col_u, smem_desc_sw128(sbase + OFF_S + koff, 16, 1024),
                                 smem_desc_sw128(sbase + OFF_W + k * 2048, 2 * TILE, 1024), ID_U, true);
                    }
                    mma_commit(&bar[B_U_FULL]);
                    // S-part of O with the unscaled Q; the chain applies gamma_r afterwards
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint32_t koff = (k >> 2) * 2 * TILE + (k & 3) * 32;
                        mma_bf16(tmem + col_o, smem_desc_sw128(sbase + OFF_S + koff, 16, 1024),
                                 smem_desc_sw128(st + TILE + koff, 16, 1024), ID_O, k > 0);
                    }
                    mma_commit(&bar[B_X_FULL]);
                    mma_commit(&bar[B_KQ_EMPTY + s]);
                    GDN_TRACE_AT(c, 2, true);
                    ++nuo;
                    issued = true;
                } else if (nwu < ng && mbar_test(&bar[B_SOLVE], nwu & 1) &&
                           mbar_test(&bar[B_V_FULL], nwu & 1) &&
                           (nwu < 1 || mbar_test(&bar[B_PREP], (nwu - 1) & 1)) &&
                           (nwu < 2 || mbar_test(&bar[u_ready(nwu)], ((nwu >> 1) - 1) & 1))) {
                    const int c = nwu, s = c & 1;
                    const uint32_t st = sbase + OFF_KQ + s * KQ_STAGE;
                    const uint32_t col_u = COL_U + s * 64;
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_bf16(tmem + COL_W, smem_desc_sw128(st + k * 2048, 2 * TILE, 1024),
                                 smem_desc_sw128(sbase + OFF_BW + k * 32, 16, 1024), ID_W, k > 0);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_bf16(tmem + col_u, smem_desc_sw128(sbase + OFF_V + k * 2048, TILE, 1024),
                                 smem_desc_sw128(sbase + OFF_BU + k * 32, 16, 1024), ID_UT, k > 0);
                    mma_commit(&bar[B_W_FULL]);
                    mma_commit(&bar[B_V_EMPTY]);
                    GDN_TRACE_AT(c, 6, true);
                    ++nwu;
                    issued = true;
                } else if (ng < nchunks && mbar_test(&bar[B_KQ_FULL + (ng & 1)], (ng >> 1) & 1) &&
                           (ng < 1 || mbar_test(&bar[B_G_FREE], (ng - 1) & 1))) {
                    const int c = ng;
                    const uint32_t st = sbase + OFF_KQ + (c & 1) * KQ_STAGE;
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint32_t koff = (k >> 2) * 2 * TILE + (k & 3) * 32;
                        mma_bf16(tmem + COL_G, smem_desc_sw128(st + koff, 16, 1024),
                                 smem_desc_sw128(st + koff, 16, 1024), ID_G, k > 0);
                    }
                    mma_commit(&bar[B_G_FULL]);
                    GDN_TRACE_AT(c, 3, true);
                    ++ng;
                    issued = true;
                }
                if (issued) {
                    idle_since = clock64();
                } else {
                    __nanosleep(64);
                    if (clock64() - idle_since > (1ll << 32)) {
                        *abort_flag = 1;
                        atomicOr(&g_tc_error, 1u);
                        break;
                    }
                }
            }
            // Drain: everything issued has completed before TMEM can be released.
            mma_commit(&bar[B_DRAIN]);
            mbar_wait(&bar[B_DRAIN], 0, 1ll << 30);
        }
    } else if (warp < 6) {
        // ======================================================== prep warpgroup
        const int pt = tid - 64;                      // 0..127
        const int q4 = warp & 3;                      // TMEM lane quarter
        const int row = q4 * 32 + lane;               // TMEM lane = matrix row
        const uint32_t t_row = tmem + ((uint32_t)(q4 * 32) << 16);
        float *sA = reinterpret_cast<float *>(sm + OFF_A);
        float *sY = reinterpret_cast<float *>(sm + OFF_Y);
        bool ok = true;
        // gate prefetch (warp 2): alpha, beta of the next chunk are in flight while
        // the current chunk is prepared
        float nx_a0 = 1.f, nx_a1 = 1.f, nx_b0 = 0.f, nx_b1 = 0.f;
        if (warp == 2 && nchunks > 0) load_gates(p, b, h, T, 0, lane, nx_a0, nx_a1, nx_b0, nx_b1);
        for (int c = 0; c < nchunks && ok; ++c) {
            const int s = c & 1;
            float *gv = reinterpret_cast<float *>(sm + OFF_GATE + s * GATE_BUF);
            GDN_TRACE_AT(c, 8, pt == 0);
#ifdef GDN_TRACE
            if (pt == 0 && blockIdx.x == 0 && blockIdx.y == 0 && c < kTraceChunks)
                g_trace[c][7] = (unsigned long long)clock64();
#endif
            // ---- gates (warp 2): b in log2 units, gamma, beta, g, beta gamma, e32;
            //      padded rows carry alpha = 1, beta = 0 (neutral)
            if (warp == 2) {
                // log2 alpha, clamped at -87 / ln 2 (alpha = 0 stays finite)
                const float la0 = fmaxf(fast_log2(nx_a0), kLog2Floor);
                const float la1 = fmaxf(fast_log2(nx_a1), kLog2Floor);
                const float be0 = nx_b0, be1 = nx_b1;
                if (c + 1 < nchunks) load_gates(p, b, h, T, c + 1, lane, nx_a0, nx_a1, nx_b0, nx_b1);
                float incl = la0 + la1;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, incl, off);
                    if (lane >= off) incl += y;
                }
                const float b0 = incl - la1, b1 = incl;
                const float blast = __shfl_sync(0xffffffffu, incl, 31);
                const float b31 = __shfl_sync(0xffffffffu, b1, 15);      // b at token 31
                const float g0 = fast_exp2(b0), g1 = fast_exp2(b1);
                gv[GV_B + 2 * lane] = b0;
                gv[GV_B + 2 * lane + 1] = b1;
                gv[GV_GAM + 2 * lane] = g0;
                gv[GV_GAM + 2 * lane + 1] = g1;
                gv[GV_BETA + 2 * lane] = be0;
                gv[GV_BETA + 2 * lane + 1] = be1;
                gv[GV_G + 2 * lane] = fast_exp2(blast - b0);
                gv[GV_G + 2 * lane + 1] = fast_exp2(blast - b1);
                gv[GV_BG + 2 * lane] = be0 * g0;
                gv[GV_BG + 2 * lane + 1] = be1 * g1;
                gv[GV_ALPHA + 2 * lane] = fast_exp2(la0);
                gv[GV_ALPHA + 2 * lane + 1] = fast_exp2(la1);
                if (lane < 16) {   // tokens 2*lane, 2*lane+1 < 32
                    gv[GV_D31 + 2 * lane] = fast_exp2(b31 - b0);
                    gv[GV_D31 + 2 * lane + 1] = fast_exp2(b31 - b1);
                }
            }
            named_sync(1, 128);
            if (pt == 0) mbar_arrive(&bar[B_GATES + s]);
            // ---- grams -> A (rows 0-63, fp32) and P (rows 64-127, bf16 operand).
            //      Decay factors Gam[r][x] = prod_{x<j<=r} alpha_j are running products
            //      along the row (no special-function work): descending from x = r,
            //      Gam[r][x-1] = Gam[r][x] alpha_x.  Rows r >= 32 continue into columns
            //      x < 32 through the table d31[x] = Gam[31][x]: Gam[r][x] = Gam[r][31] d31[x].
            //      (P buffer s is free again: the previous prep iteration waited for
            //      the last reader of that buffer, the O update of chunk c - 2.)
            ok = ctl.wait(B_KQ_FULL + s, (c >> 1) & 1) && ctl.wait(B_G_FULL, c & 1);
            ok = named_and(1, 128, ok);   // same decision in the whole warpgroup
            if (!ok) break;
            tc_fence_after();
            GDN_TRACE_AT(c, 10, pt == 0);
            {
                const int r = row & 63;
                const bool is_a = row < 64;                // A rows: strict lower; P rows: i <= r
                const bool low = r < 32;                   // warp-uniform
                float g0[32], g1[32];
                tmem_ld32(t_row + COL_G, g0);
                tmem_ld32(t_row + COL_G + 32, g1);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(&bar[B_G_FREE]);
                float run = is_a ? gv[GV_BETA + r] : 1.f;   // row scale folded into the product
                if (low) {
#pragma unroll
                    for (int x = 31; x >= 0; --x) {
                        const bool on = x <= r;
                        const bool keep = is_a ? x < r : on;
                        const float val = run * g0[x];
                        g0[x] = keep ? val : 0.f;
                        run = on ? run * gv[GV_ALPHA + x] : run;
                    }
#pragma unroll
                    for (int x = 0; x < 32; ++x) g1[x] = 0.f;
                } else {
#pragma unroll
                    for (int x = 31; x >= 0; --x) {
                        const int i = 32 + x;
                        const bool on = i <= r;
                        const bool keep = is_a ? i < r : on;
                        const float val = run * g1[x];
                        g1[x] = keep ? val : 0.f;
                        run = on ? run * gv[GV_ALPHA + i] : run;
                    }
                    // run = scale * Gam[r][31]
#pragma unroll
                    for (int x = 0; x < 32; ++x) g0[x] = run * gv[GV_D31 + x] * g0[x];
                }
                if (is_a) {
                    float4 *dst = reinterpret_cast<float4 *>(sA + r * LDA);
#pragma unroll
                    for (int x = 0; x < 8; ++x) dst[x] = make_float4(g0[4 * x], g0[4 * x + 1], g0[4 * x + 2], g0[4 * x + 3]);
#pragma unroll
                    for (int x = 0; x < 8; ++x) dst[8 + x] = make_float4(g1[4 * x], g1[4 * x + 1], g1[4 * x + 2], g1[4 * x + 3]);
                } else {
                    store_half_row_bf16(sm + OFF_P + s * TILE, r, 0, g0);
                    store_half_row_bf16(sm + OFF_P + s * TILE, r, 1, g1);
                }
            }
            named_sync(1, 128);
            GDN_TRACE_AT(c, 11, pt == 0);
            // ---- T = (I + A)^-1, then Bw = T diag(beta gamma) (threads 0-63, row pt)
            //      and Bu = T diag(beta) (threads 64-127, row pt - 64) as bf16 operands
            unit_lower_inverse(sA, sY, pt, 1);
            {
                const int r = pt & 63;
                unsigned char *dst = sm + (pt < 64 ? OFF_BW : OFF_BU);
                const float *colscale = gv + (pt < 64 ? GV_BG : GV_BETA);
#pragma unroll 1
                for (int hf = 0; hf < 2; ++hf) {
                    const float4 *trow = reinterpret_cast<const float4 *>(sA + r * LDA + 32 * hf);
                    const float4 *cs = reinterpret_cast<const float4 *>(colscale + 32 * hf);
                    float v[32];
#pragma unroll
                    for (int x = 0; x < 8; ++x) {
                        const float4 x4 = trow[x], c4 = cs[x];
                        v[4 * x] = x4.x * c4.x; v[4 * x + 1] = x4.y * c4.y;
                        v[4 * x + 2] = x4.z * c4.z; v[4 * x + 3] = x4.w * c4.w;
                    }
                    store_half_row_bf16(dst, r, hf, v);
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(&bar[B_SOLVE]);
            GDN_TRACE_AT(c, 12, pt == 0);
            // ---- W^T -> W [d][r] (MN-major B) ; K~ = diag(g) K.  The single-buffered
            //      W and K~ must no longer be read by the previous chunk's MMAs.
            ok = ctl.wait(B_W_FULL, c & 1) && (c < 1 || ctl.wait(B_U_FULL, (c - 1) & 1)) &&
                 (c < 1 || ctl.wait(B_O_FULL, (c - 1) & 1));   // also frees P of chunk c-1
            ok = named_and(1, 128, ok);
            if (!ok) break;
            tc_fence_after();
            GDN_TRACE_AT(c, 13, pt == 0);
            {
                float w0[32], w1[32];
                tmem_ld32(t_row + COL_W, w0);
                tmem_ld32(t_row + COL_W + 32, w1);
                tmem_wait_ld();
                store_half_row_bf16(sm + OFF_W, row, 0, w0);
                store_half_row_bf16(sm + OFF_W, row, 1, w1);
            }
            {
                const int i = pt >> 1, half = pt & 1;
                scale_row_bf16(sm + OFF_KQ + s * KQ_STAGE + 2 * half * TILE,
                               sm + OFF_KT + half * TILE, i, gv[GV_G + i]);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bar[B_PREP]);
            GDN_TRACE_AT(c, 14, pt == 0);
        }
    } else {
        // ======================================================== chain warpgroup
        const int q4 = warp & 3;
        const int j = q4 * 32 + lane;                 // TMEM lane = value column j
        const uint32_t t_row = tmem + ((uint32_t)(q4 * 32) << 16);
        const bool leader = (j == 0);
        bool ok = true;
        // initial state: S^T[j][d] = S0[d][j]
        {
            const float *src = p.S0 ? p.S0 + ((size_t)b * p.Hv + h) * kHeadDim * kHeadDim : nullptr;
#pragma unroll 1
            for (int c0 = 0; c0 < kHeadDim; c0 += 32) {
                float v[32];
#pragma unroll
                for (int x = 0; x < 32; ++x) v[x] = src ? src[(size_t)(c0 + x) * kHeadDim + j] : 0.f;
                tmem_st32(t_row + COL_S + c0, v);
            }
            tmem_wait_st();
        }
        for (int c = 0; c < nchunks && ok; ++c) {
            const int s = c & 1;
            GDN_TRACE_AT(c, 16, leader);
            if (c > 0) ok = ctl.wait(B_S_FULL, (c - 1) & 1);
            ok = ok && ctl.wait(B_GATES + s, (c >> 1) & 1);
            ok = named_and(2, 128, ok);
            if (!ok) break;
            tc_fence_after();
            GDN_TRACE_AT(c, 17, leader);
            const float glast = reinterpret_cast<const float *>(sm + OFF_GATE + s * GATE_BUF)[GV_GAM + C - 1];
            // S^T -> bf16 operand, and S^T <- gamma_{C-1} S^T
#pragma unroll 1
            for (int c0 = 0; c0 < kHeadDim; c0 += 64) {
                float v[64];
                tmem_ld32(t_row + COL_S + c0, v);
                tmem_ld32(t_row + COL_S + c0 + 32, v + 32);
                tmem_wait_ld();
                store_row_bf16(sm + OFF_S + (c0 >> 6) * 2 * TILE, j, v);
#pragma unroll
                for (int x = 0; x < 64; ++x) v[x] *= glast;
                tmem_st32(t_row + COL_S + c0, v);
                tmem_st32(t_row + COL_S + c0 + 32, v + 32);
            }
            tmem_wait_st();
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bar[B_S_READY]);
            GDN_TRACE_AT(c, 18, leader);
            // O epilogue of the previous chunk: O^T (lane j) -> bf16 tile [r][j] in the
            // U^T buffer (idle from the state update of c-1 to the U^T of c) -> TMA store
            if (c > 0) ok = named_and(2, 128, ctl.wait(B_O_FULL, (c - 1) & 1));
            if (!ok) break;
            if (c > 0) {
                tc_fence_after();
                const int cp = c - 1;
                const uint32_t col_o = COL_O + (cp & 1) * 64;
                unsigned char *ot = sm + OFF_U + (j >> 6) * TILE;
                const uint32_t jc = j & 63;
#pragma unroll 1
                for (int r0 = 0; r0 < C; r0 += 32) {
                    float ov[32];
                    tmem_ld32(t_row + col_o + r0, ov);
                    tmem_wait_ld();
#pragma unroll
                    for (int x = 0; x < 32; ++x)
                        *reinterpret_cast<__nv_bfloat16 *>(ot + sw128_offset(r0 + x, jc)) =
                            __float2bfloat16_rn(ov[x]);
                }
                tc_fence_before();
                mbar_arrive(&bar[B_O_FREE + (cp & 1)]);
                fence_proxy_async_smem();
                named_sync(2, 128);
                if (leader) {
                    tma_store_4d(&tm_o, sm + OFF_U, 0, h, cp * C, b);
                    tma_store_4d(&tm_o, sm + OFF_U + TILE, 64, h, cp * C, b);
                    bulk_commit_group();
                    bulk_wait_group_read0();   // staging must be read before U^T reuses it
                }
            }
            GDN_TRACE_AT(c, 19, leader);
            // U^T -> bf16 operand
            ok = ctl.wait(B_U_FULL, c & 1);
            ok = named_and(2, 128, ok);
            if (!ok) break;
            tc_fence_after();
            GDN_TRACE_AT(c, 20, leader);
            {
                float u[64];
                tmem_ld32(t_row + COL_U + s * 64, u);
                tmem_ld32(t_row + COL_U + s * 64 + 32, u + 32);
                tmem_wait_ld();
                store_row_bf16(sm + OFF_U, j, u);
            }
            // O^T S-part: column r times gamma_r (Q~ = diag(gamma) Q applied here)
            ok = named_and(2, 128, ctl.wait(B_X_FULL, c & 1));
            if (!ok) break;
            tc_fence_after();
            {
                const float *gam = reinterpret_cast<const float *>(sm + OFF_GATE + s * GATE_BUF) + GV_GAM;
                const uint32_t col_o = COL_O + s * 64;
#pragma unroll 1
                for (int r0 = 0; r0 < C; r0 += 32) {
                    float xv[32];
                    tmem_ld32(t_row + col_o + r0, xv);
                    tmem_wait_ld();
#pragma unroll
                    for (int x = 0; x < 32; ++x) xv[x] *= gam[r0 + x];
                    tmem_st32(t_row + col_o + r0, xv);
                }
                tmem_wait_st();
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bar[u_ready(c)]);
            GDN_TRACE_AT(c, 21, leader);
        }
        if (ok && nchunks > 0) {
            ok = named_and(2, 128, ctl.wait(B_O_FULL, (nchunks - 1) & 1));
            if (ok) {
                tc_fence_after();
                const int cp = nchunks - 1;
                const uint32_t col_o = COL_O + (cp & 1) * 64;
                unsigned char *ot = sm + OFF_U + (j >> 6) * TILE;
                const uint32_t jc = j & 63;
#pragma unroll 1
                for (int r0 = 0; r0 < C; r0 += 32) {
                    float ov[32];
                    tmem_ld32(t_row + col_o + r0, ov);
                    tmem_wait_ld();
#pragma unroll
                    for (int x = 0; x < 32; ++x)
                        *reinterpret_cast<__nv_bfloat16 *>(ot + sw128_offset(r0 + x, jc)) =
                            __float2bfloat16_rn(ov[x]);
                }
                fence_proxy_async_smem();
                named_sync(2, 128);
                if (leader) {
                    tma_store_4d(&tm_o, sm + OFF_U, 0, h, cp * C, b);
                    tma_store_4d(&tm_o, sm + OFF_U + TILE, 64, h, cp * C, b);
                    bulk_commit_group();
                }
            }
        }
        if (ok && p.S_final) {
            float *dst = p.S_final + ((size_t)b * p.Hv + h) * kHeadDim * kHeadDim;
#pragma unroll 1
            for (int c0 = 0; c0 < kHeadDim; c0 += 32) {
                float v[32];
                tmem_ld32(t_row + COL_S + c0, v);
                tmem_wait_ld();
#pragma unroll
                for (int x = 0; x < 32; ++x) dst[(size_t)(c0 + x) * kHeadDim + j] = v[x];
            }
        }
        if (leader) bulk_wait_group0();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ------------------------------------------------------------------ host side
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// 4-D map over a [B, T, H, 128] bf16 tensor; box = 64 head-dim x 1 head x 64 tokens x 1.
bool make_map(CUtensorMap *map, const void *base, int B, int T, int H)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)kHeadDim, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)kHeadDim * 2, (cuuint64_t)H * kHeadDim * 2,
                                   (cuuint64_t)T * H * kHeadDim * 2};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)C, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool chunk_tc_available() { return encode_fn() != nullptr; }

#ifdef GDN_TRACE
// Copies the trace of the last traced launch (kTraceChunks x kTraceSlots ns stamps).
extern "C" int gdn_trace_read(unsigned long long *host, int n)
{
    if (n < kTraceChunks * kTraceSlots) return -1;
    return (int)cudaMemcpyFromSymbol(host, g_trace, sizeof(g_trace));
}
#endif

cudaError_t launch_chunk_tc(const ChunkArgs &a, cudaStream_t stream)
{
    CUtensorMap tk, tq, tv, to;
    if (!make_map(&tk, a.k, a.B, a.T, a.Hqk) || !make_map(&tq, a.q, a.B, a.T, a.Hqk) ||
        !make_map(&tv, a.v, a.B, a.T, a.Hv) || !make_map(&to, a.o, a.B, a.T, a.Hv))
        return cudaErrorInvalidValue;
    cudaError_t err = cudaFuncSetAttribute(chunk_tc_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)SMEM_BYTES);
    if (err != cudaSuccess) return err;
    TcParams p{a.alpha, a.beta, a.S0, a.S_final, a.T, a.Hqk, a.Hv};
    chunk_tc_kernel<<<dim3((unsigned)a.Hv, (unsigned)a.B), NT, SMEM_BYTES, stream>>>(tk, tq, tv, to, p);
    return cudaGetLastError();
}

}  // namespace gdn
