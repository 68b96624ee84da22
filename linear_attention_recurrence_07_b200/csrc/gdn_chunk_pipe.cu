// Chunkwise (WY) prefill with the S-independent preparation on its own SMs:
// one cooperative launch whose CTAs take one of two roles.
//
// Source: "Qwen3.8-Flash-Next 技术总结 -- Qwen4 架构的探路者", section 2.1 "Gated
// DeltaNet": S_t = alpha_t S_{t-1} + beta_t k_t (v_t - alpha_t S_{t-1}^T k_t)^T,
// evaluated chunk by chunk with the WY representation.  Per chunk of C = 64 tokens
// (b_r = sum_{j<=r} log alpha_j, gamma_r = exp(b_r), Gam[r,i] = exp(b_r - b_i) for
// i <= r, g_i = exp(b_{C-1} - b_i)):
//   A  = strict_lower(beta_r Gam[r,i] k_r . k_i),  T = (I + A)^-1
//   W  = T diag(beta gamma) K,   U~ = T diag(beta) V,   U = U~ - W S
//   O  = diag(gamma) Q S + P U,  P = (Gam o Q K^T) masked to i <= r
//   S <- gamma_{C-1} S + (diag(g) K)^T U
// Everything before U = U~ - W S is independent of the state: the gates, the
// grams K K^T and Q K^T, A and P, the triangular inverse and the two scaled
// inverses Bw = T diag(beta gamma), Bu = T diag(beta).  That part is CUDA-core
// heavy and latency bound; the rest is a serial chain of tensor-core products
// over the chunks of one (sequence, V head).  So the two run on different SMs:
//
//   prep CTAs   one work item = one QK head group (the Hv/Hqk V heads that share
//               a QK head) x one chunk: TMA K, Q; the grams on the tensor core
//               (once per group); then one warpgroup per V head computes the
//               gates, A, P, T, Bw and Bu, and W = Bw K on the tensor core, and
//               writes W, Bu, P (bf16 operand tiles in the 128B-swizzled layout
//               the tensor core reads) and gamma, g into a ring slot in global
//               memory, then releases the slot's flag.
//   chain CTAs  one (sequence, V head) at a time, all its chunks in order: TMA
//               K, Q, V from the inputs and the ring slot from the prep; the
//               state S^T (fp32) stays in TMEM; per chunk U~^T = V^T Bu^T,
//               U^T = U~^T - S^T W^T, O^T = (S^T Q^T) diag(gamma) + U^T P^T,
//               S^T <- gamma_{C-1} S^T + (U^T diag(g)) K.  The two diagonal
//               scalings act on TMEM values (a g-scaled bf16 copy of U^T, and the
//               S-part of O^T scaled by the helper warpgroup), so the K and Q tiles
//               go to the tensor core as loaded.
//
// The ring has kRing slots per chain CTA.  A prep warpgroup writes slot n % kRing
// for the chain's n-th chunk only after the chain has loaded chunk n - kRing
// (consumed counter); the chain loads it after the slot's ready flag reads n + 1.
// Work items are issued chunk-major (all groups' chunk c before chunk c + 1), so
// the prep runs ahead of every chain by up to kRing chunks.  All CTAs are resident
// at once (cooperative launch), which the cross-CTA waits require.  Every wait is
// bounded: a wait that gives up raises a device error word and a launch-wide abort
// flag, and every CTA then drains its copies and MMAs, frees TMEM and returns.
#include <algorithm>

#include "tc_common.cuh"

namespace gdn {
namespace {

__device__ unsigned int g_pipe_error = 0;   // bit 0: a bounded wait of this kernel gave up

constexpr int NT = 512;                     // 16 warps, both roles

// Optional event trace (build with -DGDN_TRACE): %globaltimer stamps of chain CTA 0's
// roles and of the prep warpgroups that serve it, for its first kPTraceN chunks.
#ifdef GDN_TRACE
constexpr int kPTraceN = 32, kPTraceSlots = 32;
__device__ unsigned long long g_ptrace[kPTraceN][kPTraceSlots];
__device__ long long g_pclock[kPTraceN][kPTraceSlots];
__device__ __forceinline__ void ptrace(int n, int slot, bool on) {
    if (on && n >= 0 && n < kPTraceN) {
        unsigned long long t;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        g_ptrace[n][slot] = t;
        g_pclock[n][slot] = clock64();
    }
}
#ifdef GDN_TRACE_CLKONLY
#define PTRACE(n, slot, on) ((void)0)
#else
#define PTRACE(n, slot, on) ptrace((n), (slot), (on))
#endif
// whole grid: each CTA's start and end, each chain CTA's conversion start per chunk
constexpr int kGridCTAs = 160, kGridChunks = 64;
__device__ unsigned long long g_pcta[kGridCTAs][4];             // start, end, smid, SM clocks start..end
// per chain CTA and chunk: conversion start, ring flag seen, slot landed, prep release,
// S^T bf16 ready, U^T done (seen), U^T bf16 ready, O epilogue done, U~ issued, UG
// started, V load issued, V landed (seen by the U~ issuer), K/Q load issued
__device__ unsigned long long g_pchain[kGridCTAs][kGridChunks][16];
__device__ __forceinline__ unsigned long long gtimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ long long g_pclk0[kGridCTAs];
// clock64 stamps of the chain's MMA issuer: UG start / issued / done, SG start / issued /
// done (the done stamps only in builds that spin on the completion, GDN_TRACE_MMA)
__device__ long long g_pmclk[kGridCTAs][kGridChunks][24];
#define PMCLK(x, n, k) do { if ((x) < kGridCTAs && (n) < kGridChunks) g_pmclk[(x)][(n)][(k)] = clock64(); } while (0)
#define PCTA(slot) do { if (threadIdx.x == 0 && blockIdx.x < kGridCTAs) { g_pcta[blockIdx.x][(slot)] = gtimer(); \
    unsigned sid; asm volatile("mov.u32 %0, %%smid;" : "=r"(sid)); g_pcta[blockIdx.x][2] = sid; \
    if ((slot) == 0) g_pclk0[blockIdx.x] = clock64(); else g_pcta[blockIdx.x][3] = clock64() - g_pclk0[blockIdx.x]; } } while (0)
#ifdef GDN_TRACE_CLKONLY
#define PCHAIN(x, n, k, on) ((void)0)
#else
#define PCHAIN(x, n, k, on) do { if ((on) && (x) < kGridCTAs && (n) < kGridChunks) g_pchain[(x)][(n)][(k)] = gtimer(); } while (0)
#endif
// clock64 stamps inside the MMA issuer's groups (chain CTA 0, chunks 8..15)
__device__ long long g_pmma[8][24];
#define PMMA(n, slot, on) do { if ((on) && (n) >= 8 && (n) < 16) g_pmma[(n) - 8][(slot)] = clock64(); } while (0)
#else
#define PTRACE(n, slot, on) ((void)0)
#define PMMA(n, slot, on) ((void)0)
#define PCTA(slot) ((void)0)
#define PCHAIN(x, n, k, on) ((void)0)
#define PMCLK(x, n, k) ((void)0)
#endif

// ---------------------------------------------------------------- ring slot
constexpr uint32_t RS_W = 0;                          // W [d][r] bf16, MN-major B operand (16 KB)
constexpr uint32_t RS_BU = 2 * TILE, RS_P = 3 * TILE; // T diag(beta), masked decay P (8 KB each)
constexpr uint32_t RS_QT = 4 * TILE;                  // diag(gamma) Q [r][d] bf16, two d-halves (16 KB)
constexpr uint32_t RS_GATE = 6 * TILE;                // gamma[64], g[64] fp32
constexpr uint32_t RS_TILES = 6 * TILE;               // operand tiles of a slot (loaded as one copy)
constexpr uint32_t RS_GATE_BYTES = 512;               // the gate vectors (a second copy)
constexpr uint32_t RS_BYTES = 49 * 1024;              // slot stride in the ring (1024-multiple)
constexpr int kRing = 16;                             // slots per chain CTA
constexpr int kFlagWords = 32;                        // one 128-byte line per chain CTA's flags

// ---------------------------------------------------------------- chain role
constexpr uint32_t COL_S = 0;      // S^T fp32, 128 columns
constexpr uint32_t COL_SB = 128;   // S^T bf16 (64 packed columns), two buffers
constexpr uint32_t COL_U = 256;    // U^T fp32, two buffers; then U^T bf16 in place (32 packed)
constexpr uint32_t COL_O = 384;    // O^T, two buffers
constexpr uint32_t CH_TMEM_COLS = 512;

constexpr int NKQ = 3;                                // K stages, chunk n uses n % NKQ
constexpr int NRB = 3;                                // ring buffers, chunk n uses n % NRB
constexpr uint32_t KQ_STAGE = 4 * TILE;               // prep: [K d0-63][Q d0-63][K d64-127][Q d64-127]
constexpr uint32_t K_STAGE = 2 * TILE;                // chain: [K d0-63][K d64-127]
constexpr uint32_t OFF_KQ = 0;
constexpr uint32_t OFF_V = OFF_KQ + NKQ * K_STAGE;     // 2 x [V j0-63][V j64-127]
constexpr uint32_t OFF_RB = OFF_V + 4 * TILE;          // NRB ring buffers: operand tiles (32 KB each)
constexpr uint32_t OFF_RG = OFF_RB + NRB * RS_TILES;   // NRB ring buffers: gate vectors (512 B each)
constexpr uint32_t OFF_CBAR = OFF_RG + NRB * RS_GATE_BYTES;
constexpr uint32_t CH_NBAR = 40;
// named barriers of the chain CTA: the state chain (conversion warpgroups + the
// chain issuer warp), the conversion warpgroups alone, the helper warpgroup
constexpr int kChainBar = 3, kChainThreads = 288, kConvBar = 5;
constexpr uint32_t OFF_CMISC = OFF_CBAR + CH_NBAR * 8;   // TMEM base, local abort flag
constexpr uint32_t CH_SMEM_USED = OFF_CMISC + 16;
static_assert(OFF_RB % 1024 == 0 && RS_TILES % 1024 == 0 && RS_BYTES % 1024 == 0,
              "swizzled tiles need 1024-byte alignment");

// Chain CTA warps: 0 input TMA, 2 ring loader, 3 the MMA issuer off the chain,
// 4-7 and 8-11 the two conversion warpgroups (state columns 0-63 / 64-127; U
// columns 0-31 / 32-63), one thread of which issues the chain's MMAs, 12-15 the
// helper warpgroup (gamma scaling of the S-part of O, O epilogue); warp 1 idles.
enum : int {
    C_KQ_FULL = 0,    // x3 (K stage landed)
    C_KQ_EMPTY = 3,   // x3 (S and O MMAs of the chunk done: one commit of each issuer; frees
                      //     the K stage and, for U~ two chunks on, the U buffer)
    C_V_FULL = 6,     // x2
    C_V_EMPTY = 8,    // x2 (U~ MMAs done)
    C_RB_FULL = 10,   // x3 (ring slot landed)
    C_RB_EMPTY = 13,  // x3 (a commit of each issuer + the 8 conversion warps)
    C_U_FULL = 20,    // U^T done
    C_S_FULL = 23,    // state update done
    C_X_FULL = 24,    // x2 (per S^T bf16 buffer): S-part of O^T done
    C_O_FULL = 26,    // x2 O^T complete
    C_O_FREE = 28,    // x2 helper: O^T read out (4 warps)
    C_DRAIN = 30,     // both issuing threads' MMAs done (2 commits)
    C_UT_FULL = 31,   // x2 U~^T of the chunk done (its U buffer)
    C_X_GO = 33,      // x2 critical issuer: UG(n) issued (per S^T bf16 buffer)
    C_O_GO = 35,      // x2 critical issuer: SG(n) issued (per U buffer)
    C_K_FREE = 37,    // x3 helper: the O store staged in the K stage has read it
};
// Arrival counts: a tcgen05.commit counts one, a warp (warp_arrive) one.
__host__ __device__ constexpr uint32_t chain_bar_count(int i) {
    return (i >= C_RB_EMPTY && i < C_RB_EMPTY + NRB) ? 10u
         : ((i >= C_KQ_EMPTY && i < C_KQ_EMPTY + NKQ) || i == C_DRAIN) ? 2u
         : (i == C_O_FREE || i == C_O_FREE + 1) ? 4u : 1u;
}
static_assert(C_K_FREE + NKQ <= (int)CH_NBAR, "barrier count");

// ---------------------------------------------------------------- prep role
constexpr int NPKQ = 2;
constexpr int kPrepWG = 3;
constexpr uint32_t P_OFF_KQ = 0;
constexpr uint32_t P_OFF_BW = P_OFF_KQ + NPKQ * KQ_STAGE;   // per warpgroup: Bw tile (8 KB)
constexpr uint32_t P_SA = 64 * LDA * 4, P_SY = 32 * LDY * 4;
constexpr uint32_t P_WG_BYTES = P_SA + P_SY + GATE_BUF;
constexpr uint32_t P_OFF_WG = P_OFF_BW + kPrepWG * TILE;
constexpr uint32_t P_OFF_BAR = P_OFF_WG + kPrepWG * P_WG_BYTES;
constexpr uint32_t P_NBAR = 16;
constexpr uint32_t P_OFF_MISC = P_OFF_BAR + P_NBAR * 8;
constexpr uint32_t P_SMEM_USED = P_OFF_MISC + 16;
constexpr uint32_t P_TMEM_COLS = 512;   // two gram buffers (0-127), W^T per warpgroup (128 + 64 w)
enum : int {
    P_KQ_FULL = 0, P_KQ_EMPTY = 2, P_G_FULL = 4, P_G_FREE = 6,   // x2 each
    P_BW_READY = 8,   // x3 (per warpgroup): Bw tile written (4 warps)
    P_WT_FULL = 11,   // x3 (per warpgroup): W^T = K^T Bw^T done
    P_DRAIN = 14,
};
static_assert(P_WG_BYTES % 16 == 0 && P_OFF_BW % 1024 == 0, "prep shared-memory alignment");
static_assert(P_DRAIN < (int)P_NBAR, "barrier count");

constexpr uint32_t SMEM_USED = CH_SMEM_USED > P_SMEM_USED ? CH_SMEM_USED : P_SMEM_USED;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");

struct PipeParams {
    const float *alpha, *beta, *S0;
    float *S_final;
    __nv_bfloat16 *o;
    int B, T, Hqk, Hv;
    int nchunks;                  // ceil(T / 64)
    int n_chain, n_prep;          // CTA roles: blockIdx.x < n_chain is a chain CTA
    unsigned char *ring;          // [n_chain][kRing][RS_BYTES]
    unsigned *ready;              // [n_chain][kFlagWords], first kRing used: chunk counter + 1 once the slot is filled
    unsigned *consumed;           // [n_chain][kFlagWords], first used: chunks whose slot the chain has loaded
    unsigned *abort;              // launch-wide abort word (a line of its own)
    long long wait_limit;         // SM clocks a wait may take before giving up
};

__device__ __forceinline__ void st_release(unsigned *p, unsigned v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}
// Plain (non-tensor) bulk copy global -> this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ unsigned ld_relaxed(const unsigned *p) {
    unsigned v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ unsigned ld_acquire(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void fence_acquire_gpu() {
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
}

// Bounded waits that also give up once any CTA of the launch has aborted.  The
// CTA's own abort flag (shared memory) is checked on every pass; the launch-wide
// word (global memory, a round trip of about a microsecond) only every kGlobalPoll
// clocks, so that a waiting thread is never stuck in that load when its phase
// completes.
constexpr long long kGlobalPoll = 16384;
struct PCtl {
    uint64_t *bar;
    volatile int *abort_local;
    volatile unsigned *abort_global;
    long long limit;
    __device__ __forceinline__ bool aborted() const { return *abort_local != 0; }
    // Reads the launch-wide word; if another CTA aborted, marks this CTA too.
    __device__ __forceinline__ bool poll_global() const {
        if (*abort_global == 0) return false;
        *abort_local = 1;
        return true;
    }
    __device__ __noinline__ bool fail() const {
        *abort_local = 1;
        atomicOr(const_cast<unsigned *>(abort_global), 1u);
        atomicOr(&g_pipe_error, 1u);
        return false;
    }
    __device__ __forceinline__ long long poll_every() const { return limit < 4 * kGlobalPoll ? limit / 4 + 1 : kGlobalPoll; }
    // The first try inline; the bounded loop out of line (the waiting code of the
    // many call sites then costs the hot loops no instruction-cache room).
    __device__ __forceinline__ bool wait(int i, uint32_t parity) const {
        return mbar_try_wait(&bar[i], parity) || wait_loop(i, parity);
    }
    __device__ __noinline__ bool wait_loop(int i, uint32_t parity) const {
        const long long t0 = clock64();
        long long next_poll = t0 + poll_every();
        const uint32_t hint = limit < (1ll << 24) ? 200u : 20000u;
        for (;;) {
            if (mbar_try_wait_suspend(&bar[i], parity, hint)) return true;
            if (aborted()) return false;
            const long long now = clock64();
            if (now >= next_poll) {
                if (poll_global()) return false;
                next_poll = now + poll_every();
            }
            if (now - t0 > limit) return fail();
        }
    }
    // Polls a few times before falling back to wait(): for waits that usually end
    // within a few hundred clocks, where waking from a suspended try_wait is slower.
    __device__ __forceinline__ bool wait_fast(int i, uint32_t parity) const {
        return mbar_test(&bar[i], parity) || wait_fast_loop(i, parity);
    }
    __device__ __noinline__ bool wait_fast_loop(int i, uint32_t parity) const {
#pragma unroll 1
        for (int k = 0; k < 64; ++k)
            if (mbar_test(&bar[i], parity)) return true;
        return wait(i, parity);
    }
    // Waits until *p >= target (one thread; acquire once seen).  The pause between
    // polls doubles from 32 ns up to max_sleep ns, so that many waiters do not load
    // the memory system with polls while they have long to wait.
    __device__ __noinline__ bool wait_flag(const unsigned *p, unsigned target, unsigned max_sleep) const {
        if (ld_relaxed(p) >= target) { fence_acquire_gpu(); return true; }
        const long long t0 = clock64();
        long long next_poll = t0 + poll_every();
        unsigned pause = 32;
        for (;;) {
            __nanosleep(pause);
            pause = min(2 * pause, max_sleep);
            if (ld_relaxed(p) >= target) { fence_acquire_gpu(); return true; }
            if (aborted()) return false;
            const long long now = clock64();
            if (now >= next_poll) {
                if (poll_global()) return false;
                next_poll = now + poll_every();
            }
            if (now - t0 > limit) return fail();
        }
    }
    // For polling loops: true once this CTA or (checked every kGlobalPoll clocks)
    // the launch has aborted.
    __device__ __forceinline__ bool aborted_polled(long long &next_poll) const {
        if (aborted()) return true;
        const long long now = clock64();
        if (now < next_poll) return false;
        next_poll = now + poll_every();
        return poll_global();
    }
};

// alpha, beta of tokens 2*lane, 2*lane+1 of chunk cn of sequence b, V head h (alpha = 1,
// beta = 0 past the end of the sequence: those rows then add nothing to the state)
__device__ __forceinline__ void load_gates_pipe(const PipeParams &p, int b, int h, int cn, int lane,
                                                float &a0, float &a1, float &b0, float &b1) {
    const int tn = cn * C, Ln = min(C, p.T - tn);
    const int r = 2 * lane;
    const size_t gi = ((size_t)b * p.T + tn + r) * p.Hv + h;
    a0 = r < Ln ? p.alpha[gi] : 1.f;
    b0 = r < Ln ? p.beta[gi] : 0.f;
    a1 = r + 1 < Ln ? p.alpha[gi + p.Hv] : 1.f;
    b1 = r + 1 < Ln ? p.beta[gi + p.Hv] : 0.f;
}

// One arrival per warp (after the warp's lanes are done): an mbarrier serialises
// arrivals, so 128 or 256 thread arrivals would add hundreds of clocks to a hand-off.
__device__ __forceinline__ void warp_arrive(uint64_t *bar) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

// Where chunk counter n of chain CTA x lives: head wave k = n / nchunks, chunk c.
struct Unit {
    int c, b, h, hq;
};
__device__ __forceinline__ Unit unit_of(const PipeParams &p, int x, int n) {
    const int k = n / p.nchunks;
    const int hh = x + k * p.n_chain;
    Unit u;
    u.c = n - k * p.nchunks;
    u.b = hh / p.Hv;
    u.h = hh - u.b * p.Hv;
    u.hq = u.h / (p.Hv / p.Hqk);
    return u;
}
// Chunks chain CTA x processes: nchunks for each of its heads x, x + n_chain, ...
__device__ __forceinline__ int chain_units(const PipeParams &p, int x) {
    const int HH = p.B * p.Hv;
    const int heads = x < HH ? (HH - 1 - x) / p.n_chain + 1 : 0;
    return heads * p.nchunks;
}

// Rare steps of the state chain, out of line so that the per-chunk loop stays small:
// S^T[j][d] = S0[d][j] of a new head (zeros without S0), and the final state
// S_final[d][j] = S^T[j][d] of a finished one, for the thread's value column j and
// its warpgroup's 64 key dims d0 ...
__device__ __noinline__ void chain_load_s0(const float *src, uint32_t t_row, int d0, int j) {
#pragma unroll 1
    for (int c0 = d0; c0 < d0 + 64; c0 += 32) {
        float v[32];
#pragma unroll
        for (int xx = 0; xx < 32; ++xx) v[xx] = src ? src[(size_t)(c0 + xx) * kHeadDim + j] : 0.f;
        tmem_st32(t_row + COL_S + c0, v);
    }
    tmem_wait_st();
}
__device__ __noinline__ void chain_store_final(float *dst, uint32_t t_row, int d0, int j) {
#pragma unroll 1
    for (int c0 = d0; c0 < d0 + 64; c0 += 32) {
        float w[32];
        tmem_ld32(t_row + COL_S + c0, w);
        tmem_wait_ld();
#pragma unroll
        for (int xx = 0; xx < 32; ++xx) dst[(size_t)(c0 + xx) * kHeadDim + j] = w[xx];
    }
}
__device__ __noinline__ Unit unit_of_ool(const PipeParams &p, int x, int n) { return unit_of(p, x, n); }
// O rows of a chunk cut by the end of its sequence (rows < C of them exist), from the
// warp's TMEM lanes at t_col.
__device__ __noinline__ void store_o_rows(__nv_bfloat16 *dst, uint32_t t_col, int rows, size_t row_stride) {
#pragma unroll 1
    for (int r0 = 0; r0 < C; r0 += 32) {
        float ov[32];
        tmem_ld32(t_col + r0, ov);
        tmem_wait_ld();
#pragma unroll
        for (int xx = 0; xx < 32; ++xx)
            if (r0 + xx < rows) dst[(size_t)(r0 + xx) * row_stride] = __float2bfloat16_rn(ov[xx]);
    }
}

// ============================================================================ chain
__device__ __noinline__ void chain_role(const CUtensorMap *tm_k, const CUtensorMap *tm_q,
                                        const CUtensorMap *tm_v, const CUtensorMap *tm_o,
                                        const PipeParams &p, unsigned char *sm)
{
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + OFF_CBAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_CMISC);
    volatile int *abort_local = reinterpret_cast<volatile int *>(sm + OFF_CMISC + 4);
    const PCtl ctl{bar, abort_local, p.abort, p.wait_limit};
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int x = blockIdx.x;
    const int N = chain_units(p, x);
    const int nck = p.nchunks;
    const uint32_t sbase = smem_u32(sm);

    if (tid == 0) {
        prefetch_tensormap(tm_k);
        prefetch_tensormap(tm_q);
        prefetch_tensormap(tm_v);
        prefetch_tensormap(tm_o);
        for (int i = 0; i < (int)CH_NBAR; ++i) mbar_init(&bar[i], chain_bar_count(i));
        *abort_local = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, CH_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ============================================================ input TMA
        if (lane == 0) {
            int nkq = 0, nv = 0;
            long long idle_since = clock64(), next_poll = idle_since;
            while (nkq < N || nv < N) {
                if (ctl.aborted_polled(next_poll)) break;
                bool issued = false;
                if (nkq < N && (nkq < NKQ || (mbar_test(&bar[C_KQ_EMPTY + nkq % NKQ], ((nkq / NKQ) - 1) & 1) &&
                                              mbar_test(&bar[C_K_FREE + nkq % NKQ], ((nkq / NKQ) - 1) & 1)))) {
                    const Unit u = unit_of(p, x, nkq);
                    const int s = nkq % NKQ, t0 = u.c * C;
                    unsigned char *st = sm + OFF_KQ + s * K_STAGE;
                    mbar_arrive_expect_tx(&bar[C_KQ_FULL + s], K_STAGE);
                    tma_load_4d(st, tm_k, &bar[C_KQ_FULL + s], 0, u.hq, t0, u.b);
                    tma_load_4d(st + TILE, tm_k, &bar[C_KQ_FULL + s], 64, u.hq, t0, u.b);
                    PTRACE(nkq, 11, x == 0);
                    PCHAIN(x, nkq, 12, true);
                    PMCLK(x, nkq, 20);
                    ++nkq;
                    issued = true;
                }
                if (nv < N && (nv < 2 || mbar_test(&bar[C_V_EMPTY + (nv & 1)], ((nv >> 1) - 1) & 1))) {
                    const Unit u = unit_of(p, x, nv);
                    const int s = nv & 1, t0 = u.c * C;
                    unsigned char *vb = sm + OFF_V + s * 2 * TILE;
                    mbar_arrive_expect_tx(&bar[C_V_FULL + s], 2 * TILE);
                    tma_load_4d(vb, tm_v, &bar[C_V_FULL + s], 0, u.h, t0, u.b);
                    tma_load_4d(vb + TILE, tm_v, &bar[C_V_FULL + s], 64, u.h, t0, u.b);
                    PCHAIN(x, nv, 10, true);
                    ++nv;
                    issued = true;
                }
                if (issued) {
                    idle_since = clock64();
                } else {
                    __nanosleep(64);
                    if (clock64() - idle_since > p.wait_limit) {
                        ctl.fail();
                        break;
                    }
                }
            }
            if (ctl.aborted()) {   // let copies in flight land before the CTA's memory goes away:
                                   // the last load issued into each stage / buffer
                for (int m = nkq - 1; m >= 0 && m >= nkq - NKQ; --m)
                    mbar_wait(&bar[C_KQ_FULL + m % NKQ], (m / NKQ) & 1, 1ll << 28);
                for (int m = nv - 1; m >= 0 && m >= nv - 2; --m)
                    mbar_wait(&bar[C_V_FULL + (m & 1)], (m >> 1) & 1, 1ll << 28);
            }
        }
    } else if (warp == 3) {
        // ============================================================ MMA issuer (off the chain)
        //   XG(n)   O^T  = S^T Q^T      8 MMAs  after UG(n) is issued
        //   OG(n)   O^T += U^T P^T      4 MMAs  after SG(n) is issued
        //   UT(n+2) U~^T = V^T Bu^T     4 MMAs  once the S and O MMAs of n are done
        // U~ of a chunk is so computed two chunks ahead of its UG, and XG / OG queue
        // behind UG / SG in the tensor pipe.  Every barrier waited on here is one of a
        // pair (or a ring), so that no wait can miss its phase: the next phase of each
        // depends on the group the wait gates.
        if (lane == 0) {
            bool ok = true;
            auto issue_ut = [&](int n) -> bool {       // U~^T of chunk n into U buffer n & 1
                const int s = n & 1;
                if (!ctl.wait(C_V_FULL + s, (n >> 1) & 1)) return false;
                PCHAIN(x, n, 11, true);
                if (!ctl.wait(C_RB_FULL + n % NRB, (n / NRB) & 1)) return false;
                // the buffer's last readers, SG(n-2) and OG(n-2), are done
                if (n >= 2 && !ctl.wait(C_KQ_EMPTY + (n - 2) % NKQ, ((n - 2) / NKQ) & 1)) return false;
                PCHAIN(x, n, 8, true);
                tc_fence_after();
                const uint32_t vb = sbase + OFF_V + s * 2 * TILE;
                const uint32_t rb = sbase + OFF_RB + (n % NRB) * RS_TILES;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_bf16(tmem + COL_U + s * 64, smem_desc_sw128(vb + k * 2048, TILE, 1024),
                             smem_desc_sw128(rb + RS_BU + k * 32, 16, 1024), ID_UT, k > 0);
                mma_commit(&bar[C_V_EMPTY + s]);
                mma_commit(&bar[C_UT_FULL + s]);
                PTRACE(n, 2, x == 0);
                return true;
            };
            if (N > 0) ok = issue_ut(0);
            if (N > 1 && ok) ok = issue_ut(1);
            for (int n = 0; n < N && ok; ++n) {
                const int s = n & 1;
                const uint32_t rb = sbase + OFF_RB + (n % NRB) * RS_TILES;
                // XG(n): after UG(n) is issued (S^T bf16 of n written); O buffer read out
                if (!(ok = ctl.wait(C_X_GO + s, (n >> 1) & 1))) break;
                if (n >= 2 && !(ok = ctl.wait(C_O_FREE + s, ((n >> 1) - 1) & 1))) break;
                PTRACE(n, 14, x == 0);
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t koff = (k >> 2) * TILE + (k & 3) * 32;
                    mma_bf16_ts(tmem + COL_O + s * 64, tmem + COL_SB + s * 64 + k * 8,
                                smem_desc_sw128(rb + RS_QT + koff, 16, 1024), ID_O, k > 0);
                }
                mma_commit(&bar[C_X_FULL + s]);
                PTRACE(n, 15, x == 0);
                // OG(n): after SG(n) is issued (U^T bf16 of n written)
                if (!(ok = ctl.wait(C_O_GO + s, (n >> 1) & 1))) break;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_bf16_ts(tmem + COL_O + s * 64, tmem + COL_U + s * 64 + 32 * (k >> 1) + 8 * (k & 1),
                                smem_desc_sw128(rb + RS_P + k * 32, 16, 1024), ID_O, true);
                mma_commit(&bar[C_O_FULL + s]);
                mma_commit(&bar[C_RB_EMPTY + n % NRB]);
                mma_commit(&bar[C_KQ_EMPTY + n % NKQ]);
                PTRACE(n, 26, x == 0);
                // UT(n+2), ahead of its UG
                if (n + 2 < N && !(ok = issue_ut(n + 2))) break;
            }
            mma_commit(&bar[C_DRAIN]);
        }
        if (lane == 0) mbar_wait(&bar[C_DRAIN], 0, 1ll << 30);
    } else if (warp == 2) {
        // ============================================================ ring loader
        // The ready flag of chunk n is read (acquire) before waiting for its buffer,
        // so that its round trip overlaps that wait; chunk n's slot is handed back to
        // the prep (consumed counter) once its copy has landed, checked one chunk later.
        if (lane == 0) {
            const unsigned char *ring = p.ring + (size_t)x * kRing * RS_BYTES;
            const unsigned *ready = p.ready + (size_t)x * kFlagWords;
            int issued = 0;          // copies issued
            bool ok = true;
            for (int n = 0; n < N && ok; ++n) {
                const int r = n % NRB;
                PMCLK(x, n, 16);
                const unsigned flag = ld_acquire(&ready[n % kRing]);
                if (n >= NRB && !(ok = ctl.wait(C_RB_EMPTY + r, ((n / NRB) - 1) & 1))) break;
                PMCLK(x, n, 17);
                PTRACE(n, 12, x == 0);
                if (flag < (unsigned)n + 1u && !(ok = ctl.wait_flag(&ready[n % kRing], (unsigned)n + 1u, 64))) break;
                PTRACE(n, 0, x == 0);
                PCHAIN(x, n, 1, true);
                PMCLK(x, n, 18);
                fence_proxy_async_global();
                const unsigned char *src = ring + (size_t)(n % kRing) * RS_BYTES;
                mbar_arrive_expect_tx(&bar[C_RB_FULL + r], RS_TILES + RS_GATE_BYTES);
                bulk_load(sm + OFF_RB + r * RS_TILES, src, RS_TILES, &bar[C_RB_FULL + r]);
                bulk_load(sm + OFF_RG + r * RS_GATE_BYTES, src + RS_GATE, RS_GATE_BYTES, &bar[C_RB_FULL + r]);
                issued = n + 1;
                if (n >= 1) {                        // chunk n - 1's copy has landed: free its slot
                    if (!(ok = ctl.wait(C_RB_FULL + (n - 1) % NRB, ((n - 1) / NRB) & 1))) break;
                    PTRACE(n - 1, 1, x == 0);
                    PCHAIN(x, n - 1, 2, true);
                    PMCLK(x, n - 1, 19);
                    st_release(&p.consumed[(size_t)x * kFlagWords], (unsigned)n);
                }
            }
            if (ok && issued > 0 && ctl.wait(C_RB_FULL + (issued - 1) % NRB, ((issued - 1) / NRB) & 1))
                st_release(&p.consumed[(size_t)x * kFlagWords], (unsigned)issued);
            // on an abort, let the copies in flight land before the CTA's memory goes away
            for (int m = issued - 1; m >= 0 && m >= issued - NRB; --m)
                mbar_wait(&bar[C_RB_FULL + m % NRB], (m / NRB) & 1, 1ll << 28);
        }
    } else if (warp == 1) {
        // ============================================================ chain MMA issuer
        // Meets the conversion warpgroups at their named barrier (kChainBar, 288 threads:
        // 8 conversion warps and this one) and issues, right after
        //   #2 (S^T bf16 of n written):           UG(n)  U^T += S^T (-W)^T       8 MMAs
        //   #4 (U^T bf16 copies, decayed S^T):     SG(n)  S^T += (U diag(g))^T K  4 MMAs
        // The commits that release the K stage and the ring slot of n are issued after
        // UG(n+1) (they then also cover it; the last chunk's after the loop), off the
        // hand-off to the conversion.
        bool ok = true;
        for (int n = 0; n < N && ok; ++n) {
            const int s = n & 1, nk = n % NKQ, nr = n % NRB;
            const uint32_t st = sbase + OFF_KQ + nk * K_STAGE;
            const uint32_t rb = sbase + OFF_RB + nr * RS_TILES;
            bool ut_ready = false, k_ready = false;
            if (lane == 0) {
                ut_ready = mbar_test(&bar[C_UT_FULL + s], (n >> 1) & 1);
                k_ready = mbar_test(&bar[C_KQ_FULL + nk], (n / NKQ) & 1);
            }
            uint64_t wdesc[8];                        // UG's B operands, ready before the barrier
#pragma unroll
            for (int k = 0; k < 8; ++k) wdesc[k] = smem_desc_sw128(rb + RS_W + k * 2048, 2 * TILE, 1024);
            ok = named_and(kChainBar, kChainThreads, true);           // #1
            if (!ok) break;
            named_sync(kChainBar, kChainThreads);                     // #2
            if (lane == 0) {   // UG(n): its U~^T is done too
                tc_fence_after();
                if (ut_ready || ctl.wait(C_UT_FULL + s, (n >> 1) & 1)) {
                    PMCLK(x, n, 0);
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        mma_bf16_ts(tmem + COL_U + s * 64, tmem + COL_SB + s * 64 + k * 8, wdesc[k], ID_U, true);
                    PMCLK(x, n, 1);
                    mma_commit(&bar[C_U_FULL]);
#ifdef GDN_TRACE_MMA
                    for (int it = 0; it < (1 << 22) && !mbar_test(&bar[C_U_FULL], n & 1); ++it) {}
                    PMCLK(x, n, 2);
#endif
                    tc_fence_before();
                    mbar_arrive(&bar[C_X_GO + s]);
                    if (n > 0) {
                        mma_commit(&bar[C_KQ_EMPTY + (n - 1) % NKQ]);
                        mma_commit(&bar[C_RB_EMPTY + (n - 1) % NRB]);
                    }
                }
                PTRACE(n, 3, x == 0);
            }
            __syncwarp();
            ok = named_and(kChainBar, kChainThreads, true);           // #3
            if (!ok) break;
            named_sync(kChainBar, kChainThreads);                     // #4
            if (lane == 0 && (k_ready || ctl.wait(C_KQ_FULL + nk, (n / NKQ) & 1))) {
                // SG(n), once the chunk's K stage has landed (a wait that gave up leaves
                // the chunk unissued; every waiter then sees the abort)
                tc_fence_after();
                PMCLK(x, n, 3);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_bf16_ts(tmem + COL_S, tmem + COL_U + s * 64 + 32 * (k >> 1) + 16 + 8 * (k & 1),
                                smem_desc_sw128(st + k * 2048, TILE, 1024), ID_S, true);
                PMCLK(x, n, 4);
                mma_commit(&bar[C_S_FULL]);
#ifdef GDN_TRACE_MMA
                for (int it = 0; it < (1 << 22) && !mbar_test(&bar[C_S_FULL], n & 1); ++it) {}
                PMCLK(x, n, 5);
#endif
                tc_fence_before();
                mbar_arrive(&bar[C_O_GO + s]);
                PTRACE(n, 4, x == 0);
            }
            __syncwarp();
        }
        if (lane == 0) {
            if (ok && N > 0) {   // the last chunk's releases (the O epilogue waits for its K stage)
                mma_commit(&bar[C_KQ_EMPTY + (N - 1) % NKQ]);
                mma_commit(&bar[C_RB_EMPTY + (N - 1) % NRB]);
            }
            mma_commit(&bar[C_DRAIN]);
            mbar_wait(&bar[C_DRAIN], 0, 1ll << 30);
        }
    } else if (warp >= 4 && warp < 12) {
        // ============================================================ state chain
        // Two conversion warpgroups (h = 0: warps 4-7, 1: warps 8-11) own state
        // columns (key dims) 64h .. 64h+63 and U^T columns (chunk rows) 32h .. 32h+31.
        // Per chunk, with the issuer warp at the named barriers #1-#4:
        //   #1 the chunk's inputs are in: S^T -> bf16 copy;  #2 (UG issued) the decay
        //   S^T <- gamma_{C-1} S^T while UG runs (UG reads the bf16 copy);  #3 U^T done:
        //   U^T -> two bf16 copies;  #4 (SG issued).
        const int h2 = (warp - 4) >> 2;
        const int q4 = warp & 3;
        const int j = q4 * 32 + lane;                 // TMEM lane = value column j
        const uint32_t t_row = tmem + ((uint32_t)(q4 * 32) << 16);
        const bool tr0 = warp == 4 && lane == 0;      // trace stamps
        const bool has_final = p.S_final != nullptr;
        const size_t hstate = (size_t)kHeadDim * kHeadDim;
        const int d0 = 64 * h2;
        bool ok = true;
        bool pre_ready = false;                       // lane 0: X and ring tested for this chunk
        Unit u = unit_of(p, x, 0);
        for (int n = 0; n < N && ok; ++n) {
            const int s = n & 1;
            if (n > 0) {                              // the next chunk of this head, or the next head
                if (u.c + 1 < nck) ++u.c;
                else u = unit_of_ool(p, x, n);
            }
            const int nr = n % NRB;
            const float *gv = reinterpret_cast<const float *>(sm + OFF_RG + nr * RS_GATE_BYTES);
            // S^T bf16 buffer s was last read by UG(n-2) and XG(n-2); the previous
            // chunk's state update is done (for a new head: the previous head's last
            // one, whose final state was stored below); the ring slot has landed.
            // One lane per warp waits (the named barrier then orders the others after
            // it).  The first and last were usually tested already, while the
            // previous chunk's UG ran (pre_ready), so that only the state update is
            // waited for here.
            if (lane == 0) {
                if (tr0) PMCLK(x, n, 6);
                if (!pre_ready)
                    ok = ctl.wait(C_RB_FULL + nr, (n / NRB) & 1) &&
                         (n < 2 || ctl.wait(C_X_FULL + s, ((n >> 1) - 1) & 1));
                if (tr0) PMCLK(x, n, 7);
                ok = ok && (n == 0 || ctl.wait_fast(C_S_FULL, (n - 1) & 1));
                if (tr0) PMCLK(x, n, 8);
            }
            ok = named_and(kChainBar, kChainThreads, ok);             // #1
            if (!ok) break;
            tc_fence_after();
            if (tr0) PMCLK(x, n, 9);
            PTRACE(n, 5, x == 0 && j == 0 && h2 == 0);
            PCHAIN(x, n, 0, j == 0 && h2 == 0);
            if (u.c == 0)     // a new head
                chain_load_s0(p.S0 ? p.S0 + ((size_t)u.b * p.Hv + u.h) * hstate : nullptr, t_row, d0, j);
            // S^T -> packed bf16 A operand (buffer s)
            float v[64];
            {
                uint32_t pk[32];
                tmem_ld32(t_row + COL_S + d0, v);
                tmem_ld32(t_row + COL_S + d0 + 32, v + 32);
                tmem_wait_ld();
                if (tr0) PMCLK(x, n, 10);
#pragma unroll
                for (int xx = 0; xx < 32; ++xx) pk[xx] = pack_bf16x2(v[2 * xx], v[2 * xx + 1]);
                tmem_st32u(t_row + COL_SB + s * 64 + (d0 >> 1), pk);
            }
            tmem_wait_st();
            if (tr0) PMCLK(x, n, 11);
            tc_fence_before();
            named_sync(kChainBar, kChainThreads);                     // #2
            if (tr0) PMCLK(x, n, 12);
            PTRACE(n, 6, x == 0 && j == 0 && h2 == 0);
            PCHAIN(x, n, 4, j == 0 && h2 == 0);
            {   // S^T <- gamma_{C-1} S^T
                const float glast = gv[C - 1];
#pragma unroll
                for (int xx = 0; xx < 64; ++xx) v[xx] *= glast;
                tmem_st32(t_row + COL_S + d0, v);
                tmem_st32(t_row + COL_S + d0 + 32, v + 32);
            }
            // U^T (fp32, 64 columns) -> two packed bf16 copies in place, each warpgroup
            // over its own 32 columns: U^T of its 32 rows r (columns 32h .. 32h+15, for
            // the O MMAs) and (U diag(g))^T (columns 32h+16 .. 32h+31, for the state
            // update, so that K needs no scaling).
            if (tr0) PMCLK(x, n, 13);
            if (lane == 0) {   // the next chunk's ring slot and S^T bf16 buffer, while UG runs
                const int m = n + 1;
                pre_ready = m < N && mbar_test(&bar[C_RB_FULL + m % NRB], (m / NRB) & 1) &&
                            (m < 2 || mbar_test(&bar[C_X_FULL + (m & 1)], ((m >> 1) - 1) & 1));
            }
            ok = named_and(kChainBar, kChainThreads, lane != 0 || ctl.wait_fast(C_U_FULL, n & 1));   // #3
            if (!ok) break;
            if (tr0) PMCLK(x, n, 14);
            PTRACE(n, 7, x == 0 && j == 0 && h2 == 0);
            PCHAIN(x, n, 5, j == 0 && h2 == 0);
            tc_fence_after();
            {
                float uu[32];
                uint32_t pk[16];
                tmem_ld32(t_row + COL_U + s * 64 + 32 * h2, uu);
                tmem_wait_ld();
#pragma unroll
                for (int xx = 0; xx < 16; ++xx) pk[xx] = pack_bf16x2(uu[2 * xx], uu[2 * xx + 1]);
                tmem_st16u(t_row + COL_U + s * 64 + 32 * h2, pk);
                const float *gg = gv + C + 32 * h2;   // g_r of this half's rows r
#pragma unroll
                for (int xx = 0; xx < 16; ++xx)
                    pk[xx] = pack_bf16x2(uu[2 * xx] * gg[2 * xx], uu[2 * xx + 1] * gg[2 * xx + 1]);
                tmem_st16u(t_row + COL_U + s * 64 + 32 * h2 + 16, pk);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[C_RB_EMPTY + nr]);   // gates of n no longer read here
            tmem_wait_st();                       // the bf16 copies and the decayed state
            if (tr0) PMCLK(x, n, 15);
            tc_fence_before();
            named_sync(kChainBar, kChainThreads);                     // #4
            if (tr0) PMCLK(x, n, 2);
            PTRACE(n, 8, x == 0 && j == 0 && h2 == 0);
            PCHAIN(x, n, 6, j == 0 && h2 == 0);
            // last chunk of a head: store its final state once the update is done
            if (u.c == nck - 1 && has_final) {
                ok = named_and(kConvBar, 256, lane != 0 || ctl.wait(C_S_FULL, n & 1));
                if (!ok) break;
                tc_fence_after();
                chain_store_final(p.S_final + ((size_t)u.b * p.Hv + u.h) * hstate, t_row, d0, j);
                tc_fence_before();
            }
        }
    } else if (warp >= 12) {
        // ============================================================ helper warpgroup
        // The O epilogue of each chunk: O^T (TMEM) -> registers, after which the O
        // buffer is free; the bf16 tile O[r][j] goes by stmatrix into the chunk's K
        // stage (free once the chunk's S and O MMAs are done: KQ_EMPTY) and out by two
        // TMA stores; the stage returns to the K loads (C_K_FREE) once the store has
        // read it.  A chunk cut by the end of its sequence is stored row by row.
        const int pt = tid - 384;
        const int q4 = warp & 3;
        const int j = q4 * 32 + lane;
        const uint32_t t_row = tmem + ((uint32_t)(q4 * 32) << 16);
        const bool leader = pt == 0;
        const size_t row_stride = (size_t)p.Hv * kHeadDim;
        const int T = p.T;
        const int mt = lane >> 3, mi = lane & 7;
        bool ok = true;
        Unit u = unit_of(p, x, 0);
        // 16 lanes (j) x 32 columns (r) of O^T from tmem_ld16x256b_x4 -> O[r][j] bf16 in
        // the 128B-swizzled staging tiles (j 0-63, j 64-127)
        auto emit = [&](uint32_t stage, const uint32_t *rr, int sl, int cb) {
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
                uint32_t m[4];
#pragma unroll
                for (int mm = 0; mm < 4; ++mm) {
                    const int k = 2 * kk + (mm >> 1), g = mm & 1;
                    m[mm] = pack_bf16x2(__uint_as_float(rr[4 * k + 2 * g]), __uint_as_float(rr[4 * k + 2 * g + 1]));
                }
                const int k = 2 * kk + (mt >> 1), g = mt & 1;
                const int orow = 32 * cb + 8 * k + mi;
                const int jst = q4 * 32 + 16 * sl + 8 * g;
                stmatrix_x4_trans(stage + (jst >> 6) * TILE + sw128_chunk(orow, (jst & 63) >> 3), m[0], m[1], m[2], m[3]);
            }
        };
        for (int n = 0; n < N && ok; ++n) {
            const int s = n & 1, nk = n % NKQ;
            const uint32_t col_o = COL_O + s * 64;
            ok = named_and(4, 128, lane != 0 || ctl.wait(C_O_FULL + s, (n >> 1) & 1));
            if (!ok) break;
            tc_fence_after();
            if (n > 0) {                              // the next chunk of this head, or the next head
                if (u.c + 1 < nck) ++u.c;
                else u = unit_of_ool(p, x, n);
            }
            const int rows = min(C, T - u.c * C);
            if (rows == C) {
                uint32_t a0[16], b0[16], a1[16], b1[16];
                const uint32_t ta = tmem + ((uint32_t)(q4 * 32) << 16) + col_o;
                const uint32_t tb = tmem + ((uint32_t)(q4 * 32 + 16) << 16) + col_o;
                tmem_ld16x256b_x4(ta, a0);
                tmem_ld16x256b_x4(ta + 32, b0);
                tmem_ld16x256b_x4(tb, a1);
                tmem_ld16x256b_x4(tb + 32, b1);
                tmem_wait_ld();
                tc_fence_before();
                warp_arrive(&bar[C_O_FREE + s]);      // the O buffer is free once read out
                ok = named_and(4, 128, lane != 0 || ctl.wait(C_KQ_EMPTY + nk, (n / NKQ) & 1));
                if (!ok) break;
                const uint32_t stage = sbase + OFF_KQ + nk * K_STAGE;
                emit(stage, a0, 0, 0);
                emit(stage, b0, 0, 1);
                emit(stage, a1, 1, 0);
                emit(stage, b1, 1, 1);
                fence_proxy_async_smem();
                named_sync(4, 128);
                if (leader) {
                    tma_store_4d(tm_o, sm + OFF_KQ + nk * K_STAGE, 0, u.h, u.c * C, u.b);
                    tma_store_4d(tm_o, sm + OFF_KQ + nk * K_STAGE + TILE, 64, u.h, u.c * C, u.b);
                    bulk_commit_group();
                    bulk_wait_group_read0();          // the stage returns to the K loads as
                    mbar_arrive(&bar[C_K_FREE + nk]);  // soon as the store has read it
                }
            } else {
                __nv_bfloat16 *dst = p.o + ((size_t)u.b * p.T + (size_t)u.c * C) * row_stride +
                                     (size_t)u.h * kHeadDim + j;
                store_o_rows(dst, t_row + col_o, rows, row_stride);
                tc_fence_before();
                warp_arrive(&bar[C_O_FREE + s]);
                if (leader) mbar_arrive(&bar[C_K_FREE + nk]);
            }
            PTRACE(n, 10, x == 0 && j == 0);
            PCHAIN(x, n, 7, j == 0);
        }
        if (leader) bulk_wait_group0();               // the stores have read this CTA's memory
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, CH_TMEM_COLS);
    }
}

// ============================================================================ prep
// Work item i (chunk-major): wave k = i / (nchunks * groups of a full wave), then
// chunk c, then the group gi of that wave (heads k * n_chain + gi * g .. + g - 1,
// served by chain CTAs gi * g .. gi * g + g - 1 as their chunk counter k * nchunks + c).
struct Item {
    int k, c, gi, hh0;
};
__device__ __forceinline__ int groups_in_wave(const PipeParams &p, int k, int g) {
    const int HH = p.B * p.Hv;
    return min(p.n_chain, HH - k * p.n_chain) / g;
}
__device__ __forceinline__ Item item_of(const PipeParams &p, int i, int g) {
    const int full = p.n_chain / g;
    const int per_wave = p.nchunks * full;
    Item it;
    it.k = i / per_wave;
    const int rem = i - it.k * per_wave;
    const int gw = groups_in_wave(p, it.k, g);
    it.c = rem / gw;
    it.gi = rem - it.c * gw;
    it.hh0 = it.k * p.n_chain + it.gi * g;
    return it;
}
__device__ __forceinline__ int total_items(const PipeParams &p, int g) {
    const int HH = p.B * p.Hv;
    const int waves = (HH + p.n_chain - 1) / p.n_chain;
    int total = 0;
    for (int k = 0; k < waves; ++k) total += p.nchunks * groups_in_wave(p, k, g);
    return total;
}

// Prep CTA warps: 0 K/Q TMA, 1 MMA issuer (grams per item, W^T per V head), 4-15
// three V-head warpgroups (warpgroup w takes V heads w, w + 3, ... of each group).
__device__ __noinline__ void prep_role(const CUtensorMap *tm_k, const CUtensorMap *tm_q,
                                       const PipeParams &p, unsigned char *sm)
{
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + P_OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + P_OFF_MISC);
    volatile int *abort_local = reinterpret_cast<volatile int *>(sm + P_OFF_MISC + 4);
    const PCtl ctl{bar, abort_local, p.abort, p.wait_limit};
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int pidx = blockIdx.x - p.n_chain;
    const int g = p.Hv / p.Hqk;
    const int total = total_items(p, g);
    const int nmine = pidx < total ? (total - 1 - pidx) / p.n_prep + 1 : 0;   // items of this CTA
    const uint32_t sbase = smem_u32(sm);

    if (tid == 0) {
        prefetch_tensormap(tm_k);
        prefetch_tensormap(tm_q);
        for (int i = 0; i < (int)P_NBAR; ++i)
            mbar_init(&bar[i], (i == P_G_FREE || i == P_G_FREE + 1) ? 4u * kPrepWG   // warps
                               : (i >= P_BW_READY && i < P_BW_READY + kPrepWG) ? 4u : 1u);
        *abort_local = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, P_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ============================================================ K/Q loads
        if (lane == 0) {
            int nissued = 0;
            for (int jj = 0; jj < nmine; ++jj) {
                const int s = jj & 1;
                if (jj >= NPKQ && !ctl.wait(P_KQ_EMPTY + s, ((jj >> 1) - 1) & 1)) break;
                const Item it = item_of(p, pidx + jj * p.n_prep, g);
                const int b = it.hh0 / p.Hv, hq = (it.hh0 - b * p.Hv) / g, t0 = it.c * C;
                unsigned char *st = sm + P_OFF_KQ + s * KQ_STAGE;
                mbar_arrive_expect_tx(&bar[P_KQ_FULL + s], KQ_STAGE);
                tma_load_4d(st + 0 * TILE, tm_k, &bar[P_KQ_FULL + s], 0, hq, t0, b);
                tma_load_4d(st + 1 * TILE, tm_q, &bar[P_KQ_FULL + s], 0, hq, t0, b);
                tma_load_4d(st + 2 * TILE, tm_k, &bar[P_KQ_FULL + s], 64, hq, t0, b);
                tma_load_4d(st + 3 * TILE, tm_q, &bar[P_KQ_FULL + s], 64, hq, t0, b);
                nissued = jj + 1;
            }
            if (ctl.aborted())   // the last load issued into each stage
                for (int m = nissued - 1; m >= 0 && m >= nissued - NPKQ; --m)
                    mbar_wait(&bar[P_KQ_FULL + (m & 1)], (m >> 1) & 1, 1ll << 28);
        }
    } else if (warp == 1) {
        // ============================================================ MMA issuer
        // Polls for work: the grams G = [K;Q] K^T of the next item once its K/Q tiles
        // have landed and its gram buffer is free, and the W^T = K^T Bw^T product of
        // any warpgroup whose Bw tile is ready (its heads in item order).  An item's
        // K/Q stage is released after its last W^T product.
        if (lane == 0) {
            int ng = 0;                                  // items whose grams are issued
            int wt_item[kPrepWG] = {0, 0, 0};            // per warpgroup: item and head of
            int wt_head[kPrepWG] = {0, 1, 2};            //   its next W^T product
            int oldest = 0;                              // oldest item whose stage is held
            long long idle_since = clock64(), next_poll = idle_since;
            while (oldest < nmine) {
                if (ctl.aborted_polled(next_poll)) break;
                bool issued = false;
                if (ng < nmine && ng < oldest + NPKQ && mbar_test(&bar[P_KQ_FULL + (ng & 1)], (ng >> 1) & 1) &&
                    (ng < 2 || mbar_test(&bar[P_G_FREE + (ng & 1)], ((ng >> 1) - 1) & 1))) {
                    const uint32_t st = sbase + P_OFF_KQ + (ng & 1) * KQ_STAGE;
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint32_t koff = (k >> 2) * 2 * TILE + (k & 3) * 32;
                        mma_bf16(tmem + (ng & 1) * 64, smem_desc_sw128(st + koff, 16, 1024),
                                 smem_desc_sw128(st + koff, 16, 1024), ID_G, k > 0);
                    }
                    mma_commit(&bar[P_G_FULL + (ng & 1)]);
                    ++ng;
                    issued = true;
                }
#pragma unroll
                for (int w = 0; w < kPrepWG; ++w) {
                    const int jj = wt_item[w], i = wt_head[w];
                    if (jj >= nmine || jj >= ng || jj >= oldest + NPKQ) continue;
                    // the (heads_per_wg(w) * jj + i / 3)-th W^T product of warpgroup w
                    const int use = ((g - w + kPrepWG - 1) / kPrepWG) * jj + i / kPrepWG;
                    if (!mbar_test(&bar[P_BW_READY + w], use & 1)) continue;
                    const uint32_t st = sbase + P_OFF_KQ + (jj & 1) * KQ_STAGE;
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_bf16(tmem + 128 + 64 * w, smem_desc_sw128(st + k * 2048, 2 * TILE, 1024),
                                 smem_desc_sw128(sbase + P_OFF_BW + w * TILE + k * 32, 16, 1024), ID_W, k > 0);
                    mma_commit(&bar[P_WT_FULL + w]);
                    if (i + kPrepWG < g) {
                        wt_head[w] = i + kPrepWG;
                    } else {
                        wt_item[w] = jj + 1;
                        wt_head[w] = w;
                    }
                    issued = true;
                }
                // the oldest item is done once every warpgroup has moved past it
                bool past = true;
#pragma unroll
                for (int w = 0; w < kPrepWG; ++w) past = past && (w >= g || wt_item[w] > oldest);
                if (past && oldest < ng) {
                    mma_commit(&bar[P_KQ_EMPTY + (oldest & 1)]);
                    ++oldest;
                    issued = true;
                }
                if (issued) {
                    idle_since = clock64();
                } else {
                    __nanosleep(32);
                    if (clock64() - idle_since > p.wait_limit) {
                        ctl.fail();
                        break;
                    }
                }
            }
            // drain: every issued MMA has completed before TMEM is released
            mma_commit(&bar[P_DRAIN]);
            mbar_wait(&bar[P_DRAIN], 0, 1ll << 30);
        }
    } else if (warp >= 4) {
        // ============================================================ V-head warpgroups
        const int wg = (warp - 4) >> 2;               // 0 .. kPrepWG-1
        const int pt = tid - 128 - 128 * wg;          // 0 .. 127
        const int nb = 1 + wg;                        // named barrier of this warpgroup
        const int q4 = warp & 3;
        const int row = q4 * 32 + lane;               // TMEM lane = gram row (W^T: key dim d)
        const uint32_t t_row = tmem + ((uint32_t)(q4 * 32) << 16);
        unsigned char *mine = sm + P_OFF_WG + wg * P_WG_BYTES;
        float *sA = reinterpret_cast<float *>(mine);
        float *sY = reinterpret_cast<float *>(mine + P_SA);
        float *gv = reinterpret_cast<float *>(mine + P_SA + P_SY);
        unsigned char *bw_tile = sm + P_OFF_BW + wg * TILE;
        const bool gate_warp = pt < 32;
        const int heads_here = (g - wg + kPrepWG - 1) / kPrepWG;   // V heads per item on this warpgroup
        // The next head's gates (gate warp) and its ring slot's consumed counter
        // (thread 0) are loaded one head ahead, so their latency overlaps this head.
        float na0 = 1.f, na1 = 1.f, nb0 = 0.f, nb1 = 0.f;
        unsigned ncons = 0;
        auto prefetch = [&](int jj, int i) {
            if (jj >= nmine || wg >= g) return;
            const Item it = item_of(p, pidx + jj * p.n_prep, g);
            const int b = it.hh0 / p.Hv, h = it.hh0 - b * p.Hv + i;
            if (gate_warp) load_gates_pipe(p, b, h, it.c, lane, na0, na1, nb0, nb1);
            // (the first kRing chunks need no check: no load, nothing to wait for)
            if (pt == 0 && it.k * p.nchunks + it.c >= kRing)
                ncons = ld_relaxed(&p.consumed[(size_t)(it.gi * g + i) * kFlagWords]);
        };
        prefetch(0, wg);
        bool ok = true;
        for (int jj = 0; jj < nmine && ok; ++jj) {
            const int s = jj & 1;
            const Item it = item_of(p, pidx + jj * p.n_prep, g);
            const int n = it.k * p.nchunks + it.c;     // chunk counter of the chain CTAs
            PTRACE(n, 22, it.gi == 0 && pt == 0 && wg == 0);
            ok = named_and(nb, 128, ctl.wait(P_G_FULL + s, (jj >> 1) & 1));
            if (!ok) break;
            PTRACE(n, 23, it.gi == 0 && pt == 0 && wg == 0);
            tc_fence_after();
            if (wg >= g) {                            // no V head of this group here
                tc_fence_before();
                warp_arrive(&bar[P_G_FREE + s]);
                continue;
            }
            for (int i = wg; i < g && ok; i += kPrepWG) {
                const int x = it.gi * g + i;
                const bool tr = x == 0 && pt == 0;
                (void)tr;
                PTRACE(n, 16, tr);
                const float a0 = na0, a1 = na1, be0 = nb0, be1 = nb1;
                const unsigned cons = ncons;
                if (i + kPrepWG < g) prefetch(jj, i + kPrepWG);
                else prefetch(jj + 1, wg);
                // ---- the ring slot of chain CTA x for its chunk n is free once the
                //      chain has loaded chunk n - kRing
                bool free_ok = true;
                if (pt == 0 && n >= kRing) {
                    if (cons >= (unsigned)(n - kRing + 1)) fence_acquire_gpu();
                    else free_ok = ctl.wait_flag(&p.consumed[(size_t)x * kFlagWords], (unsigned)(n - kRing + 1), 256);
                }
                ok = named_and(nb, 128, free_ok);
                if (!ok) break;
                PTRACE(n, 20, tr);
                unsigned char *slot = p.ring + ((size_t)x * kRing + n % kRing) * RS_BYTES;
                // ---- gates of (b, h, chunk c)
                if (gate_warp) compute_gates(gv, a0, a1, be0, be1, lane);
                named_sync(nb, 128);
                PTRACE(n, 17, tr);
                {   // ---- Q~ = diag(gamma) Q: thread pt scales row i of d-half `half` of the
                    //      item's Q tile into the slot, in the tile layout it was loaded in
                    const int i = pt & 63, half = pt >> 6;
                    const unsigned char *qt = sm + P_OFF_KQ + s * KQ_STAGE + (2 * half + 1) * TILE;
                    scale_row_bf16(qt, slot + RS_QT + half * TILE, i, gv[GV_GAM + i]);
                }
                // ---- grams -> A rows (fp32, sA) and P rows (bf16, straight into the slot).
                //      Row r of A is beta_r Gam[r][i] k_r.k_i (i < r), of P Gam[r][i] q_r.k_i
                //      (i <= r); the decays are running products of alpha along the row from
                //      column r down (Gam[r][x-1] = Gam[r][x] alpha_x), continued into columns
                //      below 32 by d31[x] = Gam[31][x].  One 32-column half at a time: the
                //      high half first, whose running product the low half continues.
                {
                    const int r = row & 63;
                    const bool is_a = row < 64;
                    const bool low = r < 32;          // warp-uniform
                    float run = is_a ? gv[GV_BETA + r] : 1.f;
                    float gg[32];
                    tmem_ld32(t_row + s * 64 + 32, gg);
                    tmem_wait_ld();
                    if (low) {
#pragma unroll
                        for (int xx = 0; xx < 32; ++xx) gg[xx] = 0.f;
                    } else {
#pragma unroll
                        for (int xx = 31; xx >= 0; --xx) {
                            const int ci = 32 + xx;
                            const bool on = ci <= r;
                            const bool keep = is_a ? ci < r : on;
                            const float val = run * gg[xx];
                            gg[xx] = keep ? val : 0.f;
                            run = on ? run * gv[GV_ALPHA + ci] : run;
                        }
                    }
                    if (is_a) {
                        float4 *dst = reinterpret_cast<float4 *>(sA + r * LDA + 32);
#pragma unroll
                        for (int xx = 0; xx < 8; ++xx)
                            dst[xx] = make_float4(gg[4 * xx], gg[4 * xx + 1], gg[4 * xx + 2], gg[4 * xx + 3]);
                    } else {
                        store_half_row_bf16(slot + RS_P, r, 1, gg);
                    }
                    tmem_ld32(t_row + s * 64, gg);
                    tmem_wait_ld();
                    if (i + kPrepWG >= g) {           // this warpgroup's last read of the grams
                        tc_fence_before();
                        warp_arrive(&bar[P_G_FREE + s]);
                    }
                    if (low) {
#pragma unroll
                        for (int xx = 31; xx >= 0; --xx) {
                            const bool on = xx <= r;
                            const bool keep = is_a ? xx < r : on;
                            const float val = run * gg[xx];
                            gg[xx] = keep ? val : 0.f;
                            run = on ? run * gv[GV_ALPHA + xx] : run;
                        }
                    } else {                          // run = scale * Gam[r][31]
#pragma unroll
                        for (int xx = 0; xx < 32; ++xx) gg[xx] = run * gv[GV_D31 + xx] * gg[xx];
                    }
                    if (is_a) {
                        float4 *dst = reinterpret_cast<float4 *>(sA + r * LDA);
#pragma unroll
                        for (int xx = 0; xx < 8; ++xx)
                            dst[xx] = make_float4(gg[4 * xx], gg[4 * xx + 1], gg[4 * xx + 2], gg[4 * xx + 3]);
                    } else {
                        store_half_row_bf16(slot + RS_P, r, 0, gg);
                    }
                }
                named_sync(nb, 128);
                PTRACE(n, 18, tr);
                // ---- T = (I + A)^-1; Bw = T diag(beta gamma) into this warpgroup's tile
                //      (the W^T product of its previous head has read it: WT_FULL waited
                //      there), Bu = T diag(beta) into the slot
                unit_lower_inverse(sA, sY, pt, nb);
                PTRACE(n, 19, tr);
                write_bw_bu(gv, sA, pt, bw_tile, slot + RS_BU);
                fence_proxy_async_smem();
                warp_arrive(&bar[P_BW_READY + wg]);
                PTRACE(n, 25, tr);
                {
                    float *sg = reinterpret_cast<float *>(slot + RS_GATE);
                    sg[pt] = pt < 64 ? gv[GV_GAM + pt] : gv[GV_G + pt - 64];
                }
                // ---- W^T (TMEM, lane d) -> W [d][r] bf16 rows into the slot
                ok = named_and(nb, 128, ctl.wait(P_WT_FULL + wg, (heads_here * jj + i / kPrepWG) & 1));
                if (!ok) break;
                PTRACE(n, 29, tr);
                tc_fence_after();
#pragma unroll 1
                for (int half = 0; half < 2; ++half) {
                    float w0[32];
                    tmem_ld32(t_row + 128 + 64 * wg + 32 * half, w0);
                    tmem_wait_ld();
                    store_half_row_bf16(slot + RS_W, row, half, w0);
                }
                tc_fence_before();
                PTRACE(n, 30, tr);
                // every thread's slot writes come before thread 0's release (the barrier
                // orders them at CTA scope; the release is cumulative); the chain acquires
                // the flag and fences the async proxy before its bulk copy reads the slot
                named_sync(nb, 128);
                if (pt == 0) st_release(&p.ready[(size_t)x * kFlagWords + n % kRing], (unsigned)n + 1u);
                PTRACE(n, 21, tr);
                PCHAIN(x, n, 3, pt == 0);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, P_TMEM_COLS);
    }
}

__global__ void __launch_bounds__(NT, 1)
chunk_pipe_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                  const __grid_constant__ PipeParams p)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    PTRACE(0, 31, blockIdx.x == 0 && threadIdx.x == 0);
    PCTA(0);
    if ((int)blockIdx.x < p.n_chain)
        chain_role(&tm_k, &tm_q, &tm_v, &tm_o, p, sm);
    else
        prep_role(&tm_k, &tm_q, p, sm);
    PCTA(1);
}

}  // namespace
}  // namespace gdn

namespace gdn {

namespace {

// Workspace: 32-bit flag words, one 128-byte line per use (ready flags of each chain
// CTA, its consumed counter, the abort word: lines that many threads poll share no
// cache line with one another), then the ring (256-byte aligned).
constexpr size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
size_t flag_bytes(int n_chain) { return align256(((size_t)2 * n_chain + 1) * kFlagWords * sizeof(unsigned)); }

int device_sms()
{
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return sms;
}

}  // namespace

// Chain CTAs for B*Hv heads on `sms` SMs: a multiple of the QK group size g; all
// heads at once when they take at most half of the SMs, else about 60% of the SMs,
// evened out over the waves of heads.  req > 0 asks for that many (rounded down to
// a multiple of g, within [g, min(heads, sms - 1)]).
int chunk_pipe_chain_ctas(int B, int Hqk, int Hv, int sms, int req)
{
    const int g = Hv / Hqk;
    const long long HH = (long long)B * Hv;
    if (HH <= 0 || sms < 2 || g > sms - 1) return 0;
    long long cap = std::min<long long>(HH, sms - 1);
    cap -= cap % g;
    if (cap < g) return 0;
    if (req > 0) {
        long long n = std::min<long long>(req, cap);
        n -= n % g;
        return (int)std::max<long long>(n, g);
    }
    if (2 * HH <= sms) return (int)HH;
    long long n = (long long)(0.6 * sms);
    n -= n % g;
    n = std::max<long long>(std::min(n, cap), g);
    const long long waves = (HH + n - 1) / n;
    long long even = (HH + waves - 1) / waves;        // heads per wave, evened out
    even = ((even + g - 1) / g) * g;
    return (int)std::min(n, std::max<long long>(even, g));
}

size_t chunk_pipe_workspace(int B, int Hqk, int Hv)
{
    const int sms = device_sms();
    if (sms < 2 || B <= 0 || Hqk <= 0 || Hv <= 0 || Hv % Hqk) return 0;
    const int g = Hv / Hqk;
    long long cap = std::min<long long>((long long)B * Hv, sms - 1);
    cap -= cap % g;
    if (cap < g) return 0;
    return flag_bytes((int)cap) + (size_t)cap * kRing * RS_BYTES;
}

cudaError_t launch_chunk_pipe(const ChunkArgs &a, int chain_ctas, long long wait_limit,
                              void *workspace, size_t workspace_bytes, cudaStream_t stream)
{
    const int sms = device_sms();
    const int n_chain = chunk_pipe_chain_ctas(a.B, a.Hqk, a.Hv, sms, chain_ctas);
    if (n_chain <= 0) return cudaErrorInvalidValue;
    const int g = a.Hv / a.Hqk;
    const int nchunks = (a.T + C - 1) / C;
    // prep CTAs: the rest of the SMs, but no more than there are work items
    const long long HH = (long long)a.B * a.Hv;
    const long long items = nchunks * ((HH + g - 1) / g);
    const int n_prep = (int)std::min<long long>(sms - n_chain, items);
    if (n_prep < 1) return cudaErrorInvalidValue;
    const size_t fb = flag_bytes(n_chain);
    if (workspace_bytes < fb + (size_t)n_chain * kRing * RS_BYTES) return cudaErrorInvalidValue;

    static_assert(SMEM_BYTES <= 232448, "shared memory");
    cudaError_t err = cudaFuncSetAttribute(chunk_pipe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)SMEM_BYTES);
    if (err != cudaSuccess) return err;
    int per_sm = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, chunk_pipe_kernel, NT, SMEM_BYTES);
    if (err != cudaSuccess) return err;
    if ((long long)per_sm * sms < n_chain + n_prep) return cudaErrorCooperativeLaunchTooLarge;

    CUtensorMap tk, tq, tv, to;
    if (!make_map(&tk, a.k, a.B, a.T, a.Hqk) || !make_map(&tq, a.q, a.B, a.T, a.Hqk) ||
        !make_map(&tv, a.v, a.B, a.T, a.Hv) || !make_map(&to, a.o, a.B, a.T, a.Hv))
        return cudaErrorInvalidValue;
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    unsigned *flags = reinterpret_cast<unsigned *>(ws);
    err = cudaMemsetAsync(flags, 0, fb, stream);
    if (err != cudaSuccess) return err;
    PipeParams p{};
    p.alpha = a.alpha;
    p.beta = a.beta;
    p.S0 = a.S0;
    p.S_final = a.S_final;
    p.o = static_cast<__nv_bfloat16 *>(a.o);
    p.B = a.B;
    p.T = a.T;
    p.Hqk = a.Hqk;
    p.Hv = a.Hv;
    p.nchunks = nchunks;
    p.n_chain = n_chain;
    p.n_prep = n_prep;
    p.ready = flags;
    p.consumed = flags + (size_t)n_chain * kFlagWords;
    p.abort = flags + (size_t)2 * n_chain * kFlagWords;
    p.ring = ws + fb;
    p.wait_limit = wait_limit > 0 ? wait_limit : (1ll << 32);
    void *args[] = {&tk, &tq, &tv, &to, &p};
    return cudaLaunchCooperativeKernel((const void *)chunk_pipe_kernel, dim3((unsigned)(n_chain + n_prep)),
                                       dim3(NT), args, SMEM_BYTES, stream);
}

#ifdef GDN_TRACE
extern "C" int gdn_pipe_trace_read(unsigned long long *host, int n)
{
    if (n < kPTraceN * kPTraceSlots) return -1;
    return (int)cudaMemcpyFromSymbol(host, g_ptrace, sizeof(g_ptrace));
}
extern "C" int gdn_pipe_mma_read(long long *host, int n)
{
    if (n < 8 * 24) return -1;
    return (int)cudaMemcpyFromSymbol(host, g_pmma, sizeof(g_pmma));
}
extern "C" int gdn_pipe_grid_read(unsigned long long *cta, unsigned long long *chain)
{
    cudaError_t e = cudaMemcpyFromSymbol(cta, g_pcta, sizeof(g_pcta));
    if (e == cudaSuccess) e = cudaMemcpyFromSymbol(chain, g_pchain, sizeof(g_pchain));
    return (int)e;
}
extern "C" int gdn_pipe_mclk_read(long long *host)
{
    return (int)cudaMemcpyFromSymbol(host, g_pmclk, sizeof(g_pmclk));
}
extern "C" int gdn_pipe_clock_read(long long *host, int n)
{
    if (n < kPTraceN * kPTraceSlots) return -1;
    return (int)cudaMemcpyFromSymbol(host, g_pclock, sizeof(g_pclock));
}
#endif

// Reads and clears the error word of this kernel file (bit 0: a bounded wait gave up).
cudaError_t chunk_pipe_take_error(unsigned *out)
{
    unsigned v = 0, zero = 0;
    cudaError_t err = cudaMemcpyFromSymbol(&v, g_pipe_error, sizeof(v));
    if (err == cudaSuccess && v) err = cudaMemcpyToSymbol(g_pipe_error, &zero, sizeof(zero));
    *out = v;
    return err;
}

}  // namespace gdn
