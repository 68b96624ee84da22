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
//               gates, A, P, T, Bw and Bu and writes them (bf16 operand tiles in
//               the 128B-swizzled layout the tensor core reads, plus gamma and g)
//               into a ring slot in global memory, then releases the slot's flag.
//   chain CTAs  one (sequence, V head) at a time, all its chunks in order: TMA
//               K, Q, V from the inputs and the ring slot from the prep; the
//               state S^T (fp32) stays in TMEM; per chunk W^T = K^T Bw^T,
//               U~^T = V^T Bu^T, U^T = U~^T - S^T W^T, O^T = S^T Q~^T + U^T P^T,
//               S^T <- gamma_{C-1} S^T + (U^T diag(g)) K, as in the one-CTA kernel.
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

constexpr int NT = 448;                     // 14 warps, both roles

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
#define PTRACE(n, slot, on) ptrace((n), (slot), (on))
// clock64 stamps inside the MMA issuer's groups (chain CTA 0, chunks 8..15)
__device__ long long g_pmma[8][24];
#define PMMA(n, slot, on) do { if ((on) && (n) >= 8 && (n) < 16) g_pmma[(n) - 8][(slot)] = clock64(); } while (0)
#else
#define PTRACE(n, slot, on) ((void)0)
#define PMMA(n, slot, on) ((void)0)
#endif

// ---------------------------------------------------------------- ring slot
constexpr uint32_t RS_BW = 0, RS_BU = TILE, RS_P = 2 * TILE, RS_GATE = 3 * TILE;
constexpr uint32_t RS_LOAD = 3 * TILE + 512;          // bytes loaded per chunk
constexpr uint32_t RS_BYTES = 25600;                  // slot stride (1024-multiple)
constexpr int kRing = 8;                              // slots per chain CTA

// ---------------------------------------------------------------- chain role
constexpr uint32_t COL_S = 0;      // S^T fp32, 128 columns
constexpr uint32_t COL_W = 128;    // W^T fp32; after the chain read it: S^T bf16 (64 packed)
constexpr uint32_t COL_U = 192;    // U^T, two buffers; then U^T bf16 in place (32 packed)
constexpr uint32_t COL_O = 320;    // O^T, two buffers
constexpr uint32_t COL_UG = 448;   // U^T diag(g) bf16 (32 packed columns), two buffers
constexpr uint32_t CH_TMEM_COLS = 512;

constexpr int NKQ = 3;
constexpr uint32_t KQ_STAGE = 4 * TILE;               // [K d0-63][Q d0-63][K d64-127][Q d64-127]
constexpr uint32_t OFF_KQ = 0;
constexpr uint32_t OFF_V = OFF_KQ + NKQ * KQ_STAGE;    // 2 x [V j0-63][V j64-127]
constexpr uint32_t OFF_RB = OFF_V + 4 * TILE;          // 2 ring buffers (RS_BYTES each)
constexpr uint32_t OFF_W = OFF_RB + 2 * RS_BYTES;      // W stored [d][r] (MN-major B)
constexpr uint32_t OFF_OST = OFF_W + 2 * TILE;         // O staging [r][j] for the TMA store
constexpr uint32_t OFF_CBAR = OFF_OST + 2 * TILE;
constexpr uint32_t CH_NBAR = 32;
constexpr uint32_t OFF_CMISC = OFF_CBAR + CH_NBAR * 8;
constexpr uint32_t CH_SMEM_USED = OFF_CMISC + 16;
static_assert(OFF_RB % 1024 == 0 && RS_BYTES % 1024 == 0 && OFF_W % 1024 == 0 &&
              OFF_OST % 1024 == 0, "swizzled tiles need 1024-byte alignment");

enum : int {
    C_KQ_FULL = 0,    // x3
    C_KQ_EMPTY = 3,   // x3 (YS MMAs of the chunk done)
    C_V_FULL = 6,     // x2
    C_V_EMPTY = 8,    // x2 (WU MMAs done)
    C_RB_FULL = 10,   // x2 (ring slot landed)
    C_RB_EMPTY = 12,  // x2 (1 MMA commit + 128 chain + 128 helper)
    C_W_FULL = 14,    // x2 (W^T, U~^T done)
    C_S_READY = 16,   // chain: S^T bf16 in TMEM, W bf16 in SMEM (128)
    C_QT_READY = 17,  // x2 helper: Q~ scaled in place (128)
    C_U_FULL = 19,    // U^T done
    C_X_FULL = 20,    // S-part of O^T done
    C_U_READY = 21,   // x2 chain: U^T bf16 written (128)
    C_S_FULL = 23,    // state update done
    C_O_FULL = 24,    // x2 O^T complete
    C_O_FREE = 26,    // x2 helper: O^T read out (128)
    C_DRAIN = 28,
};
__host__ __device__ constexpr uint32_t chain_bar_count(int i) {
    return (i == C_RB_EMPTY || i == C_RB_EMPTY + 1) ? 257u
         : (i == C_S_READY || i == C_QT_READY || i == C_QT_READY + 1 || i == C_U_READY ||
            i == C_U_READY + 1 || i == C_O_FREE || i == C_O_FREE + 1) ? 128u : 1u;
}
static_assert(C_DRAIN < (int)CH_NBAR, "barrier count");

// ---------------------------------------------------------------- prep role
constexpr int NPKQ = 2;
constexpr int kPrepWG = 3;
constexpr uint32_t P_OFF_KQ = 0;
constexpr uint32_t P_SA = 64 * LDA * 4, P_SY = 32 * LDY * 4;
constexpr uint32_t P_WG_BYTES = P_SA + P_SY + GATE_BUF;
constexpr uint32_t P_OFF_WG = P_OFF_KQ + NPKQ * KQ_STAGE;
constexpr uint32_t P_OFF_BAR = P_OFF_WG + kPrepWG * P_WG_BYTES;
constexpr uint32_t P_NBAR = 9;
constexpr uint32_t P_OFF_MISC = P_OFF_BAR + P_NBAR * 8;
constexpr uint32_t P_SMEM_USED = P_OFF_MISC + 16;
constexpr uint32_t P_TMEM_COLS = 128;   // two gram buffers
enum : int { P_KQ_FULL = 0, P_KQ_EMPTY = 2, P_G_FULL = 4, P_G_FREE = 6, P_DRAIN = 8 };   // x2 but DRAIN
static_assert(P_WG_BYTES % 16 == 0, "per-warpgroup scratch alignment");

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
    unsigned *ready;              // [n_chain][kRing]: chunk counter + 1 once the slot is filled
    unsigned *consumed;           // [n_chain]: chunks whose slot the chain has loaded
    unsigned *abort;              // launch-wide abort word
    long long wait_limit;         // SM clocks a wait may take before giving up
};

__device__ __forceinline__ unsigned ld_acquire(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
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

// Bounded waits that also give up once any CTA of the launch has aborted.
struct PCtl {
    uint64_t *bar;
    volatile int *abort_local;
    volatile unsigned *abort_global;
    long long limit;
    __device__ __forceinline__ bool aborted() const { return *abort_local != 0 || *abort_global != 0; }
    __device__ __noinline__ bool fail() const {
        *abort_local = 1;
        atomicOr(const_cast<unsigned *>(abort_global), 1u);
        atomicOr(&g_pipe_error, 1u);
        return false;
    }
    __device__ __forceinline__ bool wait(int i, uint32_t parity) const {
        if (mbar_try_wait(&bar[i], parity)) return true;
        const long long t0 = clock64();
        const uint32_t hint = limit < (1ll << 24) ? 200u : 20000u;
        for (;;) {
            if (mbar_try_wait_suspend(&bar[i], parity, hint)) return true;
            if (aborted()) return false;
            if (clock64() - t0 > limit) return fail();
        }
    }
    // Waits until *p >= target (one thread; acquire).
    __device__ __forceinline__ bool wait_flag(const unsigned *p, unsigned target) const {
        if (ld_acquire(p) >= target) return true;
        const long long t0 = clock64();
        for (;;) {
            __nanosleep(64);
            if (ld_acquire(p) >= target) return true;
            if (aborted()) return false;
            if (clock64() - t0 > limit) return fail();
        }
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
            long long idle_since = clock64();
            while (nkq < N || nv < N) {
                if (ctl.aborted()) break;
                bool issued = false;
                if (nkq < N && (nkq < NKQ || mbar_test(&bar[C_KQ_EMPTY + nkq % NKQ], ((nkq / NKQ) - 1) & 1))) {
                    const Unit u = unit_of(p, x, nkq);
                    const int s = nkq % NKQ, t0 = u.c * C;
                    unsigned char *st = sm + OFF_KQ + s * KQ_STAGE;
                    mbar_arrive_expect_tx(&bar[C_KQ_FULL + s], KQ_STAGE);
                    tma_load_4d(st + 0 * TILE, tm_k, &bar[C_KQ_FULL + s], 0, u.hq, t0, u.b);
                    tma_load_4d(st + 1 * TILE, tm_q, &bar[C_KQ_FULL + s], 0, u.hq, t0, u.b);
                    tma_load_4d(st + 2 * TILE, tm_k, &bar[C_KQ_FULL + s], 64, u.hq, t0, u.b);
                    tma_load_4d(st + 3 * TILE, tm_q, &bar[C_KQ_FULL + s], 64, u.hq, t0, u.b);
                    PTRACE(nkq, 11, x == 0);
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
    } else if (warp == 1) {
        // ============================================================ MMA issuer
        //   YS(n): S^T += (U^T diag(g)) K, O^T += U^T P^T        needs U^T bf16 of n
        //   UO(n): U^T += S^T (-W)^T, O^T = S^T Q~^T             needs S^T bf16, W, Q~ of n
        //   WU(n): W^T = K^T Bw^T, U~^T = V^T Bu^T              needs K, V, ring slot of n
        if (lane == 0) {
            int nwu = 0, nuo = 0, nys = 0;
            long long idle_since = clock64();
            while (nys < N) {
                if (ctl.aborted()) break;
                bool issued = false;
                if (nys < nuo && mbar_test(&bar[C_U_READY + (nys & 1)], (nys >> 1) & 1)) {
                    const int n = nys, s = n & 1;
                    tc_fence_after();
                    // (compact loops: the issuing warp's code stays in the instruction cache)
                    const uint64_t bk = smem_desc_sw128(sbase + OFF_KQ + (n % NKQ) * KQ_STAGE, 2 * TILE, 1024);
#pragma unroll 1
                    for (int k = 0; k < 4; ++k)
                        mma_bf16_ts(tmem + COL_S, tmem + COL_UG + s * 32 + k * 8, bk + (uint64_t)(k * 128),
                                    ID_S, true);
                    mma_commit(&bar[C_S_FULL]);
                    mma_commit(&bar[C_KQ_EMPTY + n % NKQ]);
                    const uint64_t bp = smem_desc_sw128(sbase + OFF_RB + s * RS_BYTES + RS_P, 16, 1024);
#pragma unroll 1
                    for (int k = 0; k < 4; ++k)
                        mma_bf16_ts(tmem + COL_O + s * 64, tmem + COL_U + s * 64 + k * 8, bp + (uint64_t)(k * 2),
                                    ID_O, true);
                    mma_commit(&bar[C_O_FULL + s]);
                    mma_commit(&bar[C_RB_EMPTY + s]);
                    PTRACE(n, 4, x == 0);
                    ++nys;
                    issued = true;
                } else if (nuo < nwu && mbar_test(&bar[C_S_READY], nuo & 1) &&
                           mbar_test(&bar[C_QT_READY + (nuo & 1)], (nuo >> 1) & 1) &&
                           (nuo < 2 || mbar_test(&bar[C_O_FREE + (nuo & 1)], ((nuo >> 1) - 1) & 1))) {
                    const int n = nuo, s = n & 1;
                    const uint32_t st = sbase + OFF_KQ + (n % NKQ) * KQ_STAGE;
                    tc_fence_after();
                    const uint64_t bw = smem_desc_sw128(sbase + OFF_W, 2 * TILE, 1024);
                    PMMA(n, 0, x == 0);
#pragma unroll 1
                    for (int k = 0; k < 8; ++k) {
                        mma_bf16_ts(tmem + COL_U + s * 64, tmem + COL_W + k * 8, bw + (uint64_t)(k * 128), ID_U, true);
                        PMMA(n, 1 + k, x == 0);
                    }
                    mma_commit(&bar[C_U_FULL]);
                    PMMA(n, 9, x == 0);
                    const uint64_t bq = smem_desc_sw128(st + TILE, 16, 1024);
#pragma unroll 1
                    for (int k = 0; k < 8; ++k) {
                        mma_bf16_ts(tmem + COL_O + s * 64, tmem + COL_W + k * 8,
                                    bq + (uint64_t)(((k >> 2) * 2 * TILE + (k & 3) * 32) >> 4), ID_O, k > 0);
                        PMMA(n, 10 + k, x == 0);
                    }
                    mma_commit(&bar[C_X_FULL]);
                    PMMA(n, 18, x == 0);
                    PTRACE(n, 3, x == 0);
                    ++nuo;
                    issued = true;
                } else if (nwu < N && mbar_test(&bar[C_KQ_FULL + nwu % NKQ], (nwu / NKQ) & 1) &&
                           mbar_test(&bar[C_V_FULL + (nwu & 1)], (nwu >> 1) & 1) &&
                           mbar_test(&bar[C_RB_FULL + (nwu & 1)], (nwu >> 1) & 1) &&
                           // UO of n-1 (last reader of the S^T bf16 in the W^T columns) done;
                           // so are the YS MMAs of n-2 (readers of this U^T buffer), issued before it
                           (nwu < 1 || mbar_test(&bar[C_X_FULL], (nwu - 1) & 1))) {
                    const int n = nwu, s = n & 1;
                    const uint32_t st = sbase + OFF_KQ + (n % NKQ) * KQ_STAGE;
                    const uint32_t rb = sbase + OFF_RB + s * RS_BYTES;
                    const uint32_t vb = sbase + OFF_V + s * 2 * TILE;
                    tc_fence_after();
                    const uint64_t ak = smem_desc_sw128(st, 2 * TILE, 1024);
                    const uint64_t bbw = smem_desc_sw128(rb + RS_BW, 16, 1024);
#pragma unroll 1
                    for (int k = 0; k < 4; ++k)
                        mma_bf16(tmem + COL_W, ak + (uint64_t)(k * 128), bbw + (uint64_t)(k * 2), ID_W, k > 0);
                    const uint64_t av = smem_desc_sw128(vb, TILE, 1024);
                    const uint64_t bbu = smem_desc_sw128(rb + RS_BU, 16, 1024);
#pragma unroll 1
                    for (int k = 0; k < 4; ++k)
                        mma_bf16(tmem + COL_U + s * 64, av + (uint64_t)(k * 128), bbu + (uint64_t)(k * 2), ID_UT, k > 0);
                    mma_commit(&bar[C_W_FULL + s]);
                    mma_commit(&bar[C_V_EMPTY + s]);
                    PTRACE(n, 2, x == 0);
                    ++nwu;
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
            mma_commit(&bar[C_DRAIN]);
            mbar_wait(&bar[C_DRAIN], 0, 1ll << 30);
        }
    } else if (warp == 2) {
        // ============================================================ ring loader
        if (lane == 0) {
            const unsigned char *ring = p.ring + (size_t)x * kRing * RS_BYTES;
            const unsigned *ready = p.ready + (size_t)x * kRing;
            int pending = -1;        // a load issued but not yet seen landed
            for (int n = 0; n < N; ++n) {
                const int s = n & 1;
                if (n >= 2 && !ctl.wait(C_RB_EMPTY + s, ((n >> 1) - 1) & 1)) break;
                PTRACE(n, 12, x == 0);
                if (!ctl.wait_flag(&ready[n % kRing], (unsigned)n + 1u)) break;
                PTRACE(n, 0, x == 0);
                fence_proxy_async_global();
                mbar_arrive_expect_tx(&bar[C_RB_FULL + s], RS_LOAD);
                bulk_load(sm + OFF_RB + s * RS_BYTES, ring + (size_t)(n % kRing) * RS_BYTES, RS_LOAD,
                          &bar[C_RB_FULL + s]);
                pending = n;
                if (!ctl.wait(C_RB_FULL + s, (n >> 1) & 1)) break;
                pending = -1;
                PTRACE(n, 1, x == 0);
                st_release(&p.consumed[x], (unsigned)n + 1u);   // the slot may be refilled
            }
            if (pending >= 0) mbar_wait(&bar[C_RB_FULL + (pending & 1)], (pending >> 1) & 1, 1ll << 28);
        }
    } else if (warp >= 4 && warp < 8) {
        // ============================================================ helper warpgroup
        // Q~ = diag(gamma) Q in place for the UO MMAs, and the O epilogue (TMEM ->
        // bf16 tile [r][j] by stmatrix -> one TMA store per chunk; row stores for a
        // chunk cut by the end of the sequence).
        const int pt = tid - 128;
        const int q4 = warp & 3;
        const int j = q4 * 32 + lane;
        const uint32_t t_row = tmem + ((uint32_t)(q4 * 32) << 16);
        const bool leader = pt == 0;
        const size_t row_stride = (size_t)p.Hv * kHeadDim;
        bool ok = true;
        auto epilogue = [&](int n) -> bool {
            if (leader) bulk_wait_group_read0();     // the previous store has read the staging tile
            if (!named_and(1, 128, ctl.wait(C_O_FULL + (n & 1), (n >> 1) & 1))) return false;
            tc_fence_after();
            const Unit u = unit_of(p, x, n);
            const uint32_t col_o = COL_O + (n & 1) * 64;
            const int rows = min(C, p.T - u.c * C);
            if (rows == C) {
                const uint32_t stage = smem_u32(sm + OFF_OST);
                const int mt = lane >> 3, mi = lane & 7;
                auto emit = [&](const uint32_t *rr, int sl, int cb) {
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk) {
                        uint32_t m[4];
#pragma unroll
                        for (int mm = 0; mm < 4; ++mm) {
                            const int k = 2 * kk + (mm >> 1), g = mm & 1;
                            m[mm] = pack_bf16x2(__uint_as_float(rr[4 * k + 2 * g]),
                                                __uint_as_float(rr[4 * k + 2 * g + 1]));
                        }
                        const int k = 2 * kk + (mt >> 1), g = mt & 1;
                        const int orow = 32 * cb + 8 * k + mi;
                        const int jst = q4 * 32 + 16 * sl + 8 * g;
                        stmatrix_x4_trans(stage + (jst >> 6) * TILE + sw128_chunk(orow, (jst & 63) >> 3),
                                          m[0], m[1], m[2], m[3]);
                    }
                };
#pragma unroll 1
                for (int sl = 0; sl < 2; ++sl) {
                    uint32_t ra[16], rb[16];
                    const uint32_t ta = tmem + ((uint32_t)(q4 * 32 + 16 * sl) << 16) + col_o;
                    tmem_ld16x256b_x4(ta, ra);
                    tmem_ld16x256b_x4(ta + 32, rb);
                    tmem_wait_ld();
                    emit(ra, sl, 0);
                    emit(rb, sl, 1);
                }
                tc_fence_before();
                mbar_arrive(&bar[C_O_FREE + (n & 1)]);
                fence_proxy_async_smem();
                named_sync(1, 128);
                if (leader) {
                    tma_store_4d(tm_o, sm + OFF_OST, 0, u.h, u.c * C, u.b);
                    tma_store_4d(tm_o, sm + OFF_OST + TILE, 64, u.h, u.c * C, u.b);
                    bulk_commit_group();
                }
                return true;
            }
            __nv_bfloat16 *dst = p.o + ((size_t)u.b * p.T + (size_t)u.c * C) * row_stride +
                                 (size_t)u.h * kHeadDim + j;
#pragma unroll 1
            for (int r0 = 0; r0 < C; r0 += 32) {
                float ov[32];
                tmem_ld32(t_row + col_o + r0, ov);
                tmem_wait_ld();
#pragma unroll
                for (int xx = 0; xx < 32; ++xx)
                    if (r0 + xx < rows) dst[(size_t)(r0 + xx) * row_stride] = __float2bfloat16_rn(ov[xx]);
            }
            tc_fence_before();
            mbar_arrive(&bar[C_O_FREE + (n & 1)]);
            return true;
        };
        for (int n = 0; n < N && ok; ++n) {
            const int s = n & 1;
            ok = ctl.wait(C_KQ_FULL + n % NKQ, (n / NKQ) & 1) && ctl.wait(C_RB_FULL + s, (n >> 1) & 1);
            ok = named_and(1, 128, ok);
            if (!ok) break;
            {
                const float *gam = reinterpret_cast<const float *>(sm + OFF_RB + s * RS_BYTES + RS_GATE);
                const int i = pt >> 1, half = pt & 1;
                unsigned char *qt = sm + OFF_KQ + (n % NKQ) * KQ_STAGE + (2 * half + 1) * TILE;
                scale_row_bf16(qt, qt, i, gam[i]);
            }
            fence_proxy_async_smem();
            PTRACE(n, 9, x == 0 && pt == 0);
            mbar_arrive(&bar[C_QT_READY + s]);
            mbar_arrive(&bar[C_RB_EMPTY + s]);
            if (n > 0 && !(ok = epilogue(n - 1))) break;
            PTRACE(n - 1, 10, x == 0 && pt == 0);
        }
        if (ok && N > 0) ok = epilogue(N - 1);
        if (leader) bulk_wait_group0();
    } else if (warp >= 8 && warp < 12) {
        // ============================================================ chain warpgroup
        const int q4 = warp & 3;
        const int j = q4 * 32 + lane;                 // TMEM lane = value column j (W^T: key dim d)
        const uint32_t t_row = tmem + ((uint32_t)(q4 * 32) << 16);
        const size_t hstate = (size_t)kHeadDim * kHeadDim;
        bool ok = true;
        for (int n = 0; n < N && ok; ++n) {
            const int s = n & 1;
            const Unit u = unit_of(p, x, n);
            const float *gv = reinterpret_cast<const float *>(sm + OFF_RB + s * RS_BYTES + RS_GATE);
            // W^T (TMEM, lane d) -> W [d][r] bf16 (MN-major B of the U MMAs); the U MMAs
            // of n-1, the last readers of the W tile, have completed (U_FULL, waited in n-1)
            ok = named_and(2, 128, ctl.wait(C_W_FULL + s, (n >> 1) & 1));
            if (!ok) break;
            PTRACE(n, 5, x == 0 && j == 0);
            tc_fence_after();
            {
                float w0[32], w1[32];
                tmem_ld32(t_row + COL_W, w0);
                tmem_ld32(t_row + COL_W + 32, w1);
                tmem_wait_ld();
                store_half_row_bf16(sm + OFF_W, j, 0, w0);
                store_half_row_bf16(sm + OFF_W, j, 1, w1);
            }
            // the previous chunk's state update is done (for a new head: the previous
            // head's last one, whose final state was stored below)
            if (n > 0) ok = ctl.wait(C_S_FULL, (n - 1) & 1);
            ok = ok && ctl.wait(C_RB_FULL + s, (n >> 1) & 1);
            ok = named_and(2, 128, ok);
            if (!ok) break;
            tc_fence_after();
            if (u.c == 0) {   // a new head: S^T[j][d] = S0[d][j] (zeros without S0)
                const float *src = p.S0 ? p.S0 + ((size_t)u.b * p.Hv + u.h) * hstate : nullptr;
#pragma unroll 1
                for (int c0 = 0; c0 < kHeadDim; c0 += 32) {
                    float v[32];
#pragma unroll
                    for (int xx = 0; xx < 32; ++xx) v[xx] = src ? src[(size_t)(c0 + xx) * kHeadDim + j] : 0.f;
                    tmem_st32(t_row + COL_S + c0, v);
                }
                tmem_wait_st();
            }
            // S^T -> packed bf16 A operand in the (read) W^T columns; S^T <- gamma_{C-1} S^T
            const float glast = gv[C - 1];
#pragma unroll 1
            for (int c0 = 0; c0 < kHeadDim; c0 += 32) {
                float v[32];
                uint32_t pk[16];
                tmem_ld32(t_row + COL_S + c0, v);
                tmem_wait_ld();
#pragma unroll
                for (int xx = 0; xx < 16; ++xx) pk[xx] = pack_bf16x2(v[2 * xx], v[2 * xx + 1]);
                tmem_st16u(t_row + COL_W + (c0 >> 1), pk);
#pragma unroll
                for (int xx = 0; xx < 32; ++xx) v[xx] *= glast;
                tmem_st32(t_row + COL_S + c0, v);
            }
            tmem_wait_st();
            fence_proxy_async_smem();                // the W tile, for the tensor core
            tc_fence_before();
            mbar_arrive(&bar[C_S_READY]);
            PTRACE(n, 6, x == 0 && j == 0);
            // U^T -> packed bf16 A operands in place: U^T (columns 0-31 of its buffer)
            // for the O update, U^T diag(g) (columns 32-63) for the state update
            ok = named_and(2, 128, ctl.wait(C_U_FULL, n & 1));
            if (!ok) break;
            PTRACE(n, 7, x == 0 && j == 0);
            tc_fence_after();
#pragma unroll 1
            for (int c0 = 0; c0 < C; c0 += 32) {   // packed U^T in place: writes trail reads
                float uu[32];
                uint32_t pk[16];
                tmem_ld32(t_row + COL_U + s * 64 + c0, uu);
                tmem_wait_ld();
#pragma unroll
                for (int xx = 0; xx < 16; ++xx) pk[xx] = pack_bf16x2(uu[2 * xx], uu[2 * xx + 1]);
                tmem_st16u(t_row + COL_U + s * 64 + (c0 >> 1), pk);
                const float4 *g4 = reinterpret_cast<const float4 *>(gv + C + c0);
#pragma unroll
                for (int xx = 0; xx < 8; ++xx) {
                    const float4 g = g4[xx];
                    pk[2 * xx] = pack_bf16x2(uu[4 * xx] * g.x, uu[4 * xx + 1] * g.y);
                    pk[2 * xx + 1] = pack_bf16x2(uu[4 * xx + 2] * g.z, uu[4 * xx + 3] * g.w);
                }
                tmem_st16u(t_row + COL_UG + s * 32 + (c0 >> 1), pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bar[C_U_READY + s]);
            mbar_arrive(&bar[C_RB_EMPTY + s]);      // gamma, g of n no longer read
            PTRACE(n, 8, x == 0 && j == 0);
            // last chunk of a head: store its final state once the update is done
            if (u.c == nck - 1 && p.S_final) {
                ok = named_and(2, 128, ctl.wait(C_S_FULL, n & 1));
                if (!ok) break;
                tc_fence_after();
                float *dst = p.S_final + ((size_t)u.b * p.Hv + u.h) * hstate;
#pragma unroll 1
                for (int c0 = 0; c0 < kHeadDim; c0 += 32) {
                    float v[32];
                    tmem_ld32(t_row + COL_S + c0, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int xx = 0; xx < 32; ++xx) dst[(size_t)(c0 + xx) * kHeadDim + j] = v[xx];
                }
                tc_fence_before();
            }
        }
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
            mbar_init(&bar[i], (i == P_G_FREE || i == P_G_FREE + 1) ? 128u * kPrepWG : 1u);
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
        // ============================================================ grams
        if (lane == 0) {
            for (int jj = 0; jj < nmine; ++jj) {
                const int s = jj & 1;
                if (!ctl.wait(P_KQ_FULL + s, (jj >> 1) & 1)) break;
                if (jj >= 2 && !ctl.wait(P_G_FREE + s, ((jj >> 1) - 1) & 1)) break;
                tc_fence_after();
                const uint32_t st = sbase + P_OFF_KQ + s * KQ_STAGE;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t koff = (k >> 2) * 2 * TILE + (k & 3) * 32;
                    mma_bf16(tmem + s * 64, smem_desc_sw128(st + koff, 16, 1024),
                             smem_desc_sw128(st + koff, 16, 1024), ID_G, k > 0);
                }
                mma_commit(&bar[P_G_FULL + s]);
                mma_commit(&bar[P_KQ_EMPTY + s]);
            }
            // drain: every issued MMA has completed before TMEM is released
            mma_commit(&bar[P_DRAIN]);
            mbar_wait(&bar[P_DRAIN], 0, 1ll << 30);
        }
    } else if (warp >= 2) {
        // ============================================================ V-head warpgroups
        // (warps 2-5, 6-9, 10-13: each four consecutive warps, one per TMEM lane quarter)
        const int wg = (warp - 2) >> 2;               // 0 .. kPrepWG-1
        const int pt = tid - 64 - 128 * wg;           // 0 .. 127
        const int nb = 1 + wg;                        // named barrier of this warpgroup
        const int q4 = warp & 3;
        const int row = q4 * 32 + lane;               // TMEM lane = gram row
        const uint32_t t_row = tmem + ((uint32_t)(q4 * 32) << 16);
        unsigned char *mine = sm + P_OFF_WG + wg * P_WG_BYTES;
        float *sA = reinterpret_cast<float *>(mine);
        float *sY = reinterpret_cast<float *>(mine + P_SA);
        float *gv = reinterpret_cast<float *>(mine + P_SA + P_SY);
        const bool gate_warp = pt < 32;
        bool ok = true;
        for (int jj = 0; jj < nmine && ok; ++jj) {
            const int s = jj & 1;
            const Item it = item_of(p, pidx + jj * p.n_prep, g);
            const int b = it.hh0 / p.Hv, h0 = it.hh0 - b * p.Hv;
            const int n = it.k * p.nchunks + it.c;     // chunk counter of the chain CTAs
            PTRACE(n, 22, it.gi == 0 && pt == 0 && wg == 0);
            ok = named_and(nb, 128, ctl.wait(P_G_FULL + s, (jj >> 1) & 1));
            if (!ok) break;
            PTRACE(n, 23, it.gi == 0 && pt == 0 && wg == 0);
            tc_fence_after();
            if (wg >= g) {                            // no V head of this group here
                tc_fence_before();
                mbar_arrive(&bar[P_G_FREE + s]);
                continue;
            }
            for (int i = wg; i < g && ok; i += kPrepWG) {
                const int h = h0 + i, x = it.gi * g + i;
                const bool tr = x == 0 && pt == 0;
                PTRACE(n, 16, tr);
                // ---- the ring slot of chain CTA x for its chunk n is free once the
                //      chain has loaded chunk n - kRing
                bool free_ok = true;
                if (pt == 0 && n >= kRing) free_ok = ctl.wait_flag(&p.consumed[x], (unsigned)(n - kRing + 1));
                ok = named_and(nb, 128, free_ok);
                if (!ok) break;
                PTRACE(n, 20, tr);
                unsigned char *slot = p.ring + ((size_t)x * kRing + n % kRing) * RS_BYTES;
                // ---- gates of (b, h, chunk c)
                if (gate_warp) {
                    float a0, a1, b0, b1;
                    load_gates_pipe(p, b, h, it.c, lane, a0, a1, b0, b1);
                    compute_gates(gv, a0, a1, b0, b1, lane);
                }
                named_sync(nb, 128);
                PTRACE(n, 17, tr);
                // ---- grams -> A rows (fp32, sA) and P rows (bf16, straight into the slot)
                {
                    float g0[32], g1[32];
                    tmem_ld32(t_row + s * 64, g0);
                    tmem_ld32(t_row + s * 64 + 32, g1);
                    tmem_wait_ld();
                    if (i + kPrepWG >= g) {           // this warpgroup's last read of the grams
                        tc_fence_before();
                        mbar_arrive(&bar[P_G_FREE + s]);
                    }
                    ap_row_values(gv, row, g0, g1);
                    if (row < 64) {
                        float4 *dst = reinterpret_cast<float4 *>(sA + row * LDA);
#pragma unroll
                        for (int xx = 0; xx < 8; ++xx)
                            dst[xx] = make_float4(g0[4 * xx], g0[4 * xx + 1], g0[4 * xx + 2], g0[4 * xx + 3]);
#pragma unroll
                        for (int xx = 0; xx < 8; ++xx)
                            dst[8 + xx] = make_float4(g1[4 * xx], g1[4 * xx + 1], g1[4 * xx + 2], g1[4 * xx + 3]);
                    } else {
                        store_half_row_bf16(slot + RS_P, row - 64, 0, g0);
                        store_half_row_bf16(slot + RS_P, row - 64, 1, g1);
                    }
                }
                named_sync(nb, 128);
                PTRACE(n, 18, tr);
                // ---- T = (I + A)^-1
                unit_lower_inverse(sA, sY, pt, nb);
                PTRACE(n, 19, tr);
                write_bw_bu(gv, sA, pt, slot + RS_BW, slot + RS_BU);
                {
                    float *sg = reinterpret_cast<float *>(slot + RS_GATE);
                    sg[pt] = pt < 64 ? gv[GV_GAM + pt] : gv[GV_G + pt - 64];
                }
                fence_proxy_async_global();
                named_sync(nb, 128);
                if (pt == 0) {
                    __threadfence();
                    st_release(&p.ready[(size_t)x * kRing + n % kRing], (unsigned)n + 1u);
                }
                PTRACE(n, 21, tr);
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
    if ((int)blockIdx.x < p.n_chain)
        chain_role(&tm_k, &tm_q, &tm_v, &tm_o, p, sm);
    else
        prep_role(&tm_k, &tm_q, p, sm);
}

}  // namespace
}  // namespace gdn

namespace gdn {

namespace {

// Workspace: [ready: n_chain * kRing][consumed: n_chain][abort] as 32-bit words,
// then the ring (256-byte aligned).
constexpr size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
size_t flag_bytes(int n_chain) { return align256(((size_t)n_chain * (kRing + 1) + 1) * sizeof(unsigned)); }

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
    p.consumed = flags + (size_t)n_chain * kRing;
    p.abort = flags + (size_t)n_chain * (kRing + 1);
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
