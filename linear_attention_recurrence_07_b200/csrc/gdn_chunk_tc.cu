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
//   O^T  = S^T Q~^T + U^T P^T,  Q~ = diag(gamma) Q,  P = masked Gam o Q K^T
//   S^T <- gamma_{C-1} S^T + U^T K~,  K~ = diag(g) K                   M=128 N=128 K=64
// The state S^T (128 lanes x 128 fp32 columns) stays in TMEM for the whole
// sequence; its bf16 copy in shared memory is only an MMA operand.
//
// One CTA per (sequence, V head), warp-specialised, two chunks in flight:
//   warp 0      TMA producer: K, Q (double-buffered) and V tiles, 128B swizzle
//   warp 1      MMA issuer (one thread)
//   warps 2-5   "prep" warpgroup, one chunk ahead of the state: gates, A and P
//               from the grams, the triangular solve (fp32, CUDA cores), W^T to
//               shared memory, Q~ and K~
//   warps 6-9   "chain" warpgroup, the state-dependent path: S^T -> bf16
//               operand (+ decay of the fp32 state), U^T -> bf16 operand, and
//               the O epilogue of the previous chunk
// The state-dependent critical path per chunk is two MMA groups and two
// TMEM -> shared-memory conversions; the rest overlaps with it.
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
constexpr uint32_t COL_U = 256;    // U^T
constexpr uint32_t COL_O = 320;    // O^T, two buffers (320, 384)
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
constexpr uint32_t OFF_U = OFF_S + 4 * TILE;      // U^T bf16 [j][i]
constexpr uint32_t OFF_AT = OFF_U + 2 * TILE;     // A split by row parity: At[h][col][row/2], fp32
constexpr uint32_t AT_HALF = 64 * 32 * 4 + 16;    // 8 KiB + 16 B so the halves use other banks
constexpr uint32_t OFF_GATE = OFF_AT + 2 * AT_HALF;  // 2 buffers x {b2, gamma, beta, g} x 64
constexpr uint32_t GATE_BUF = 4 * C * 4;
constexpr uint32_t OFF_BAR = OFF_GATE + 2 * GATE_BUF;
constexpr uint32_t NBAR = 20;
constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;    // tmem slot, abort flag
constexpr uint32_t SMEM_USED = OFF_MISC + 16;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;    // slack for aligning the base

// barrier indices
enum : int {
    B_KQ_FULL = 0,   // 2: TMA K/Q stage landed
    B_KQ_EMPTY = 2,  // 2: stage no longer read
    B_V_FULL = 4, B_V_EMPTY = 5,
    B_G_FULL = 6,    // grams done
    B_W_FULL = 7,    // W^T, U~^T done
    B_SOLVE = 8,     // prep: Bw, Bu, P, Q~ written (128 arrivals)
    B_PREP = 9,      // prep: W, K~ written (128 arrivals)
    B_GATES = 10,    // 2: gates of a chunk written (1 arrival)
    B_S_READY = 12,  // chain: S^T bf16 written (128)
    B_U_FULL = 13,   // U^T and S-part of O done
    B_U_READY = 14,  // chain: U^T bf16 written (128)
    B_S_FULL = 15,   // state update and O done
    B_O_FREE = 16,   // 2: O accumulator read out (128)
    B_DRAIN = 18,    // final MMA drain
};

constexpr uint32_t ID_G = idesc_bf16(128, 64, false, false);
constexpr uint32_t ID_W = idesc_bf16(128, 64, true, false);
constexpr uint32_t ID_UT = idesc_bf16(128, 64, true, false);
constexpr uint32_t ID_U = idesc_bf16(128, 64, false, true, /*neg_b=*/true);
constexpr uint32_t ID_O = idesc_bf16(128, 64, false, false);
constexpr uint32_t ID_S = idesc_bf16(128, 128, false, true);

constexpr float kLog2e = 1.4426950408889634f;

struct TcParams {
    const float *alpha, *beta, *S0;
    __nv_bfloat16 *o;
    float *S_final;
    int T, Hqk, Hv;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// 64 fp32 values (one row, times `scale`) -> bf16 row `row` of a 128B-swizzled tile.
__device__ __forceinline__ void store_row_bf16(unsigned char *tile, uint32_t row, const float *x,
                                               float scale = 1.f) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        uint4 v;
        v.x = pack_bf16x2(x[8 * c + 0] * scale, x[8 * c + 1] * scale);
        v.y = pack_bf16x2(x[8 * c + 2] * scale, x[8 * c + 3] * scale);
        v.z = pack_bf16x2(x[8 * c + 4] * scale, x[8 * c + 5] * scale);
        v.w = pack_bf16x2(x[8 * c + 6] * scale, x[8 * c + 7] * scale);
        *reinterpret_cast<uint4 *>(tile + sw128_chunk(row, c)) = v;
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
                const __grid_constant__ CUtensorMap tm_v, const TcParams p)
{
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
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
        for (int i = 0; i < (int)NBAR; ++i) {
            const bool many = (i == B_SOLVE || i == B_PREP || i == B_S_READY || i == B_U_READY ||
                               i == B_O_FREE || i == B_O_FREE + 1);
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
            int issued_kq[2] = {-1, -1}, issued_v = -1;
            for (int c = 0; c < nchunks && ok; ++c) {
                const int s = c & 1, t0 = c * C;
                if (c >= 2) ok = ctl.wait(B_KQ_EMPTY + s, ((c >> 1) - 1) & 1);
                if (!ok) break;
                unsigned char *st = sm + OFF_KQ + s * KQ_STAGE;
                GDN_TRACE_AT(c, 24, true);
                mbar_arrive_expect_tx(&bar[B_KQ_FULL + s], KQ_STAGE);
                tma_load_4d(st + 0 * TILE, &tm_k, &bar[B_KQ_FULL + s], 0, hq, t0, b);
                tma_load_4d(st + 1 * TILE, &tm_q, &bar[B_KQ_FULL + s], 0, hq, t0, b);
                tma_load_4d(st + 2 * TILE, &tm_k, &bar[B_KQ_FULL + s], 64, hq, t0, b);
                tma_load_4d(st + 3 * TILE, &tm_q, &bar[B_KQ_FULL + s], 64, hq, t0, b);
                issued_kq[s] = c;
                if (c >= 1) ok = ctl.wait(B_V_EMPTY, (c - 1) & 1);
                if (!ok) break;
                mbar_arrive_expect_tx(&bar[B_V_FULL], 2 * TILE);
                tma_load_4d(sm + OFF_V, &tm_v, &bar[B_V_FULL], 0, h, t0, b);
                tma_load_4d(sm + OFF_V + TILE, &tm_v, &bar[B_V_FULL], 64, h, t0, b);
                issued_v = c;
                GDN_TRACE_AT(c, 25, true);
            }
            if (*abort_flag) {
                // Let copies still in flight land before the CTA's memory goes away.
                for (int s = 0; s < 2; ++s)
                    if (issued_kq[s] >= 0) mbar_wait(&bar[B_KQ_FULL + s], (issued_kq[s] >> 1) & 1, 1ll << 28);
                if (issued_v >= 0) mbar_wait(&bar[B_V_FULL], issued_v & 1, 1ll << 28);
            }
        }
    } else if (warp == 1) {
        // ======================================================== MMA issuer
        if (lane == 0) {
            bool ok = true;
            auto issue_g = [&](int c) {
                const uint32_t st = sbase + OFF_KQ + (c & 1) * KQ_STAGE;
#pragma unroll
                for (int s = 0; s < 8; ++s) {
                    const uint32_t koff = (s >> 2) * 2 * TILE + (s & 3) * 32;
                    mma_bf16(tmem + COL_G, smem_desc_sw128(st + koff, 16, 1024),
                             smem_desc_sw128(st + koff, 16, 1024), ID_G, s > 0);
                }
                mma_commit(&bar[B_G_FULL]);
            };
            auto issue_wu = [&](int c) {
                const uint32_t st = sbase + OFF_KQ + (c & 1) * KQ_STAGE;
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_bf16(tmem + COL_W, smem_desc_sw128(st + s * 2048, 2 * TILE, 1024),
                             smem_desc_sw128(sbase + OFF_BW + s * 32, 16, 1024), ID_W, s > 0);
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_bf16(tmem + COL_U, smem_desc_sw128(sbase + OFF_V + s * 2048, TILE, 1024),
                             smem_desc_sw128(sbase + OFF_BU + s * 32, 16, 1024), ID_UT, s > 0);
                mma_commit(&bar[B_W_FULL]);
                mma_commit(&bar[B_V_EMPTY]);
            };
            if (nchunks > 0) {
                ok = ctl.wait(B_KQ_FULL, 0);
                if (ok) { tc_fence_after(); issue_g(0); }
                ok = ok && ctl.wait(B_SOLVE, 0) && ctl.wait(B_V_FULL, 0);
                if (ok) { tc_fence_after(); issue_wu(0); }
            }
            for (int c = 0; c < nchunks && ok; ++c) {
                const int s = c & 1;
                const uint32_t st = sbase + OFF_KQ + s * KQ_STAGE;
                const uint32_t col_o = COL_O + s * 64;
                GDN_TRACE_AT(c, 0, true);
                ok = ctl.wait(B_PREP, c & 1) && ctl.wait(B_S_READY, c & 1);
                if (ok && c >= 2) ok = ctl.wait(B_O_FREE + s, ((c >> 1) - 1) & 1);
                if (!ok) break;
                GDN_TRACE_AT(c, 1, true);
                tc_fence_after();
                // U^T += S^T (-W)^T ; O^T = S^T Q~^T
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t koff = (k >> 2) * 2 * TILE + (k & 3) * 32;
                    mma_bf16(tmem + COL_U, smem_desc_sw128(sbase + OFF_S + koff, 16, 1024),
                             smem_desc_sw128(sbase + OFF_W + k * 2048, 2 * TILE, 1024), ID_U, true);
                }
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t koff = (k >> 2) * 2 * TILE + (k & 3) * 32;
                    mma_bf16(tmem + col_o, smem_desc_sw128(sbase + OFF_S + koff, 16, 1024),
                             smem_desc_sw128(st + TILE + koff, 16, 1024), ID_O, k > 0);
                }
                mma_commit(&bar[B_U_FULL]);
                mma_commit(&bar[B_KQ_EMPTY + s]);
                GDN_TRACE_AT(c, 2, true);
                // grams of the next chunk
                if (c + 1 < nchunks) {
                    ok = ctl.wait(B_KQ_FULL + ((c + 1) & 1), ((c + 1) >> 1) & 1);
                    if (!ok) break;
                    tc_fence_after();
                    issue_g(c + 1);
                    GDN_TRACE_AT(c, 3, true);
                }
                // O^T += U^T P^T ; S^T += U^T K~
                ok = ctl.wait(B_U_READY, c & 1);
                if (!ok) break;
                GDN_TRACE_AT(c, 4, true);
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_bf16(tmem + col_o, smem_desc_sw128(sbase + OFF_U + k * 32, 16, 1024),
                             smem_desc_sw128(sbase + OFF_P + s * TILE + k * 32, 16, 1024), ID_O, true);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_bf16(tmem + COL_S, smem_desc_sw128(sbase + OFF_U + k * 32, 16, 1024),
                             smem_desc_sw128(sbase + OFF_KT + k * 2048, TILE, 1024), ID_S, true);
                mma_commit(&bar[B_S_FULL]);
                GDN_TRACE_AT(c, 5, true);
                // W^T and U~^T of the next chunk
                if (c + 1 < nchunks) {
                    ok = ctl.wait(B_SOLVE, (c + 1) & 1) && ctl.wait(B_V_FULL, (c + 1) & 1);
                    if (!ok) break;
                    GDN_TRACE_AT(c, 6, true);
                    tc_fence_after();
                    issue_wu(c + 1);
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
        const int cc = (pt >> 5) * 16 + (lane & 15);  // solve: column of T
        const int hp = lane >> 4;                     // solve: row parity owned
        float *At0 = reinterpret_cast<float *>(sm + OFF_AT);
        float *At1 = reinterpret_cast<float *>(sm + OFF_AT + AT_HALF);
        float *At_mine = hp ? At1 : At0;
        bool ok = true;
        // gate prefetch (warp 2): alpha, beta of the next chunk are in flight while
        // the current chunk is prepared
        float nx_a[2] = {1.f, 1.f}, nx_b[2] = {0.f, 0.f};
        auto load_gates = [&](int cn) {
            const int tn = cn * C, Ln = min(C, T - tn);
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                const int r = 2 * lane + x;
                const size_t gi = ((size_t)b * T + tn + r) * p.Hv + h;
                nx_a[x] = r < Ln ? p.alpha[gi] : 1.f;
                nx_b[x] = r < Ln ? p.beta[gi] : 0.f;
            }
        };
        if (warp == 2 && nchunks > 0) load_gates(0);
        for (int c = 0; c < nchunks && ok; ++c) {
            const int s = c & 1, t0 = c * C, L = min(C, T - t0);
            float *gb = reinterpret_cast<float *>(sm + OFF_GATE + s * GATE_BUF);
            float *s_b2 = gb, *s_gam = gb + C, *s_beta = gb + 2 * C, *s_g = gb + 3 * C;
            GDN_TRACE_AT(c, 8, pt == 0);
            // ---- gates (warp 2): b in log2 units, gamma, beta, g; padded rows neutral
            if (warp == 2) {
                // padded rows carry alpha = 1, beta = 0 (neutral)
                const float la[2] = {clamped_log(nx_a[0]) * kLog2e, clamped_log(nx_a[1]) * kLog2e};
                const float be[2] = {nx_b[0], nx_b[1]};
                if (c + 1 < nchunks) load_gates(c + 1);
                float incl = la[0] + la[1];
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, incl, off);
                    if (lane >= off) incl += y;
                }
                const float b0 = incl - la[1], b1 = incl;
                const float blast = __shfl_sync(0xffffffffu, incl, 31);
                s_b2[2 * lane] = b0;
                s_b2[2 * lane + 1] = b1;
                s_gam[2 * lane] = fast_exp2(b0);
                s_gam[2 * lane + 1] = fast_exp2(b1);
                s_beta[2 * lane] = be[0];
                s_beta[2 * lane + 1] = be[1];
                s_g[2 * lane] = fast_exp2(blast - b0);
                s_g[2 * lane + 1] = fast_exp2(blast - b1);
            }
            named_sync(1, 128);
            GDN_TRACE_AT(c, 9, pt == 0);
            if (pt == 0) mbar_arrive(&bar[B_GATES + s]);
            // ---- grams -> A (rows 0-63, stored split by row parity, transposed) and P
            ok = ctl.wait(B_KQ_FULL + s, (c >> 1) & 1) && ctl.wait(B_G_FULL, c & 1);
            ok = named_and(1, 128, ok);   // same decision in the whole warpgroup
            if (!ok) break;
            GDN_TRACE_AT(c, 10, pt == 0);
            tc_fence_after();
            {
                float g[64];
                tmem_ld32(t_row + COL_G, g);
                tmem_ld32(t_row + COL_G + 32, g + 32);
                tmem_wait_ld();
                const int r = row & 63;
                const float br = s_b2[r];
                if (row < 64) {
                    const float be = s_beta[r];
                    float *dst = (r & 1 ? At1 : At0) + (r >> 1);
#pragma unroll
                    for (int i = 0; i < C; ++i)
                        dst[i * 32] = i < r ? be * fast_exp2(br - s_b2[i]) * g[i] : 0.f;
                } else {
#pragma unroll
                    for (int i = 0; i < C; ++i) g[i] = i <= r ? fast_exp2(br - s_b2[i]) * g[i] : 0.f;
                    store_row_bf16(sm + OFF_P + s * TILE, r, g);
                }
            }
            // Q~ = diag(gamma) Q, in place in the stage (the grams have consumed Q)
            {
                const int i = pt >> 1, half = pt & 1;
                unsigned char *qt = sm + OFF_KQ + s * KQ_STAGE + (1 + 2 * half) * TILE;
                scale_row_bf16(qt, qt, i, s_gam[i]);
            }
            tc_fence_before();
            named_sync(1, 128);
            GDN_TRACE_AT(c, 11, pt == 0);
            // ---- T = (I + A)^-1, column cc; this thread owns the rows of parity hp.
            //      Right-looking: once x_r is final, subtract A[r', r] x_r from later rows.
            {
                float x[32];
#pragma unroll
                for (int m = 0; m < 32; ++m) x[m] = (2 * m + hp == cc) ? 1.f : 0.f;
                const int src_base = lane & 15;
#pragma unroll
                for (int r = 0; r < C - 1; ++r) {
                    const float xr = __shfl_sync(0xffffffffu, x[r >> 1], src_base | ((r & 1) << 4));
                    const float4 *arow = reinterpret_cast<const float4 *>(At_mine + r * 32);
                    // rows 2m + hp > r  <=>  m >= (r + 1 - hp + 1) / 2 ; start at a multiple of 4
#pragma unroll
                    for (int m4 = (r >> 1) >> 2; m4 < 8; ++m4) {
                        const float4 a = arow[m4];
                        x[4 * m4 + 0] = fmaf(-a.x, xr, x[4 * m4 + 0]);
                        x[4 * m4 + 1] = fmaf(-a.y, xr, x[4 * m4 + 1]);
                        x[4 * m4 + 2] = fmaf(-a.z, xr, x[4 * m4 + 2]);
                        x[4 * m4 + 3] = fmaf(-a.w, xr, x[4 * m4 + 3]);
                    }
                }
                const float sw = s_beta[cc] * s_gam[cc], su = s_beta[cc];
#pragma unroll
                for (int m = 0; m < 32; ++m) {
                    const uint32_t off = sw128_offset(2 * m + hp, cc);
                    *reinterpret_cast<__nv_bfloat16 *>(sm + OFF_BW + off) = __float2bfloat16_rn(x[m] * sw);
                    *reinterpret_cast<__nv_bfloat16 *>(sm + OFF_BU + off) = __float2bfloat16_rn(x[m] * su);
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(&bar[B_SOLVE]);
            GDN_TRACE_AT(c, 12, pt == 0);
            // ---- W^T -> W [d][r] (MN-major B) ; K~ = diag(g) K
            ok = named_and(1, 128, ctl.wait(B_W_FULL, c & 1));
            if (!ok) break;
            GDN_TRACE_AT(c, 13, pt == 0);
            tc_fence_after();
            {
                float w[64];
                tmem_ld32(t_row + COL_W, w);
                tmem_ld32(t_row + COL_W + 32, w + 32);
                tmem_wait_ld();
                store_row_bf16(sm + OFF_W, row, w);
            }
            {
                const int i = pt >> 1, half = pt & 1;
                scale_row_bf16(sm + OFF_KQ + s * KQ_STAGE + 2 * half * TILE,
                               sm + OFF_KT + half * TILE, i, s_g[i]);
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
        auto epilogue = [&](int cprev) {
            // O of chunk cprev: O[r][j] from O^T lane j -> global (rows inside the sequence)
            const int t0 = cprev * C, L = min(C, T - t0);
            const uint32_t col_o = COL_O + (cprev & 1) * 64;
            __nv_bfloat16 *dst = p.o + (((size_t)b * T + t0) * p.Hv + h) * kHeadDim + j;
            const size_t rstride = (size_t)p.Hv * kHeadDim;
#pragma unroll 1
            for (int r0 = 0; r0 < C; r0 += 32) {
                float ov[32];
                tmem_ld32(t_row + col_o + r0, ov);
                tmem_wait_ld();
#pragma unroll
                for (int x = 0; x < 32; ++x)
                    if (r0 + x < L) dst[(size_t)(r0 + x) * rstride] = __float2bfloat16_rn(ov[x]);
            }
            tc_fence_before();
            mbar_arrive(&bar[B_O_FREE + (cprev & 1)]);
        };
        for (int c = 0; c < nchunks && ok; ++c) {
            const int s = c & 1;
            GDN_TRACE_AT(c, 16, j == 0);
            if (c > 0) ok = ctl.wait(B_S_FULL, (c - 1) & 1);
            ok = ok && ctl.wait(B_GATES + s, (c >> 1) & 1);
            ok = __all_sync(0xffffffffu, ok);   // tcgen05.ld/st below are warp-collective
            if (!ok) break;
            GDN_TRACE_AT(c, 17, j == 0);
            tc_fence_after();
            const float glast = reinterpret_cast<const float *>(sm + OFF_GATE + s * GATE_BUF)[C + C - 1];
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
            GDN_TRACE_AT(c, 18, j == 0);
            if (c > 0) epilogue(c - 1);
            GDN_TRACE_AT(c, 19, j == 0);
            // U^T -> bf16 operand
            ok = __all_sync(0xffffffffu, ctl.wait(B_U_FULL, c & 1));
            if (!ok) break;
            GDN_TRACE_AT(c, 20, j == 0);
            tc_fence_after();
            {
                float u[64];
                tmem_ld32(t_row + COL_U, u);
                tmem_ld32(t_row + COL_U + 32, u + 32);
                tmem_wait_ld();
                store_row_bf16(sm + OFF_U, j, u);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bar[B_U_READY]);
            GDN_TRACE_AT(c, 21, j == 0);
        }
        if (ok && nchunks > 0) {
            ok = __all_sync(0xffffffffu, ctl.wait(B_S_FULL, (nchunks - 1) & 1));
            if (ok) {
                tc_fence_after();
                epilogue(nchunks - 1);
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
    CUtensorMap tk, tq, tv;
    if (!make_map(&tk, a.k, a.B, a.T, a.Hqk) || !make_map(&tq, a.q, a.B, a.T, a.Hqk) ||
        !make_map(&tv, a.v, a.B, a.T, a.Hv))
        return cudaErrorInvalidValue;
    cudaError_t err = cudaFuncSetAttribute(chunk_tc_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)SMEM_BYTES);
    if (err != cudaSuccess) return err;
    TcParams p{a.alpha, a.beta, a.S0, (__nv_bfloat16 *)a.o, a.S_final, a.T, a.Hqk, a.Hv};
    chunk_tc_kernel<<<dim3((unsigned)a.Hv, (unsigned)a.B), NT, SMEM_BYTES, stream>>>(tk, tq, tv, p);
    return cudaGetLastError();
}

}  // namespace gdn
