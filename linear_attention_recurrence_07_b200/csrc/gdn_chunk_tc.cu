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
//   S^T <- gamma_{C-1} S^T + (U^T diag(g)) K                            M=128 N=128 K=64
// The state S^T (128 lanes x 128 fp32 columns) stays in TMEM for the whole
// sequence.  The two state-side A operands, S^T and U^T, go to the tensor core
// from TMEM as packed bf16 (written by the chain with tcgen05.st): they never
// touch shared memory, whose bandwidth the operand reads of the other MMAs and
// the CUDA-core prep work already share.
//
// One CTA per (sequence, V head), warp-specialised:
//   warp 0      TMA producer: K, Q (three stages) and V tiles, 128B swizzle
//   warp 1      MMA issuer (one thread), event-driven: it issues whichever MMA
//               group has its inputs ready, state-dependent groups first
//   warps 2-9   two "prep" warpgroups (even / odd chunks), running ahead of the
//               state: gates, A and P from the grams, the triangular solve (fp32
//               CUDA cores + TF32 warp MMAs for the block merges), Bw, Bu, and
//               Q~ = diag(gamma) Q in place
//   warps 10-13 "chain" warpgroup, the state-dependent path: W^T -> bf16 W
//               operand (shared memory), S^T -> bf16 A operand in TMEM (+ decay
//               of the fp32 state), U^T -> two bf16 A operands in TMEM (in place:
//               U^T for the O update, U^T diag(g) for the state update), and
//               the O epilogue (O^T blocks transposed into a bf16 tile staged in
//               the idle W tile by stmatrix, one TMA store per chunk)
// TMEM columns are reused: the bf16 S^T takes the W^T columns once W^T has been
// read, the two bf16 copies of U^T the two halves of its own fp32 buffer.  The U^T and O^T
// accumulators are double-buffered, so the prep work of the next chunk never
// waits for the state-dependent chain of the current one.
//
// Every wait is bounded.  On a timeout the CTA raises a device error flag, the
// other roles see a shared abort flag and stop, in-flight copies and MMAs are
// drained (again with a bound) and TMEM is freed before returning.
#include "tc_common.cuh"

namespace gdn {

namespace {

constexpr int NT = 448;            // 14 warps

// TMEM columns (fp32 accumulators over 128 lanes)
constexpr uint32_t COL_S = 0;      // S^T: 128 columns
constexpr uint32_t COL_G = 128;    // [K;Q] K^T
constexpr uint32_t COL_W = 192;    // W^T; after the chain read it: S^T bf16 (64 packed columns)
constexpr uint32_t COL_U = 256;    // U^T, two buffers (256, 320); then U^T, U^T diag(g) bf16 (32 + 32)
constexpr uint32_t COL_O = 384;    // O^T, two buffers (384, 448)
constexpr uint32_t TMEM_COLS = 512;

// Shared-memory plan (byte offsets from a 1024-aligned base).
constexpr int NKQ = 3;                            // K/Q stages, chunk c uses c % NKQ
constexpr uint32_t OFF_KQ = 0;                    // NKQ stages x [K d0-63][Q d0-63][K d64-127][Q d64-127]
constexpr uint32_t KQ_STAGE = 4 * TILE;
constexpr uint32_t OFF_V = OFF_KQ + NKQ * KQ_STAGE;  // [V j0-63][V j64-127]
constexpr uint32_t OFF_P = OFF_V + 2 * TILE;      // 2 x P [r][i] K-major
constexpr uint32_t OFF_BW = OFF_P + 2 * TILE;     // T diag(beta gamma) [r][i]
constexpr uint32_t OFF_BU = OFF_BW + TILE;        // T diag(beta)       [r][i]
constexpr uint32_t OFF_W = OFF_BU + TILE;         // W stored [d][r] (MN-major B), 128 rows
constexpr uint32_t SA_BYTES = 64 * LDA * 4, SY_BYTES = 32 * LDY * 4;
constexpr uint32_t OFF_A = OFF_W + 2 * TILE;      // 2 x A, then T = (I + A)^-1, fp32 [64][LDA]
constexpr uint32_t OFF_Y = OFF_A + 2 * SA_BYTES;  // 2 x solve scratch, fp32 [32][LDY]
constexpr int NGATE = 3;                          // gate buffers, chunk c uses c % NGATE
constexpr uint32_t OFF_GATE = OFF_Y + 2 * SY_BYTES;
constexpr uint32_t OFF_BAR = OFF_GATE + NGATE * GATE_BUF;
constexpr uint32_t NBAR = 34;
constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;    // tmem slot, abort flag
constexpr uint32_t SMEM_USED = OFF_MISC + 16;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;    // slack for aligning the base
static_assert(OFF_V % 1024 == 0 && OFF_W % 1024 == 0, "swizzled tiles need 1024-byte alignment");
static_assert(OFF_GATE % 16 == 0 && GATE_BUF % 16 == 0, "gate vectors are read as float4");
static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");

// Barrier indices (arrival count 1 unless noted).  "x2" barriers are per chunk
// parity (chunk c uses index c & 1), "x3" per gate buffer (c % 3): a role that
// waits for chunk c - 2 (or c - 3) while another chunk's phase may already have
// completed on a shared barrier would read the wrong phase, so every barrier that
// such a role waits on completes once per chunk of its own class, in order.
enum : int {
    B_KQ_FULL = 0,   // x3 (per K/Q stage): TMA K/Q stage landed
    B_KQ_EMPTY = 3,  // x3: stage no longer read (after the state update)
    B_V_FULL = 6, B_V_EMPTY = 7,
    B_G_FULL = 8,    // x2: grams done
    B_W_FULL = 10,   // x2: W^T, U~^T done
    B_SOLVE = 12,    // x2: prep: Bw, Bu written, the K of its stage read (128)
    B_PREP = 14,     // x2: prep: P written (128)
    B_GATES = 16,    // x3: gates of a chunk written
    B_GFREE = 19,    // x3: chain: gates of a chunk no longer read (128)
    B_S_READY = 22,  // chain: S^T bf16 (TMEM) and W bf16 written (128)
    B_U_FULL = 23,   // U^T done
    B_U_READY = 24,  // x2: chain: U^T bf16 (TMEM) written, O^T scaled (128)
    B_S_FULL = 26,   // state update done
    B_O_FREE = 27,   // x2: O accumulator read out (128)
    B_DRAIN = 29,    // final MMA drain
    B_G_FREE = 30,   // prep: grams read out of TMEM (128)
    B_X_FULL = 31,   // S-part of O^T (S^T Q^T) done
    B_O_FULL = 32,   // x2: O^T complete (after U^T P^T)
};
__host__ __device__ constexpr int u_ready(int c) { return B_U_READY + (c & 1); }
__host__ __device__ constexpr bool many_arrivals(int i) {
    return i == B_SOLVE || i == B_SOLVE + 1 || i == B_PREP || i == B_PREP + 1 ||
           (i >= B_GFREE && i < B_GFREE + NGATE) || i == B_S_READY || i == B_U_READY ||
           i == B_U_READY + 1 || i == B_O_FREE || i == B_O_FREE + 1 || i == B_G_FREE;
}
static_assert(B_O_FULL + 2 <= (int)NBAR, "barrier count");

// Bounded waits for this kernel: the first try inline, the loop out of line, so
// that the waiting code of the many call sites costs the per-chunk loops no
// instruction-cache room.  A wait that gives up raises the abort flag and the
// device error word; every role then stops.
struct TcCtl {
    uint64_t *bar;
    volatile int *abort_flag;
    __device__ __forceinline__ bool wait(int i, uint32_t parity) const {
        return mbar_try_wait(&bar[i], parity) || wait_loop(i, parity);
    }
    __device__ __noinline__ bool wait_loop(int i, uint32_t parity) const {
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

// O rows of a chunk cut by the end of its sequence (rows < C exist), from the
// warp's TMEM lanes at t_col; out of line (rare).
__device__ __noinline__ void tc_store_o_rows(__nv_bfloat16 *dst, uint32_t t_col, int rows, size_t row_stride) {
#pragma unroll 1
    for (int r0 = 0; r0 < C; r0 += 32) {
        float ov[32];
        tmem_ld32(t_col + r0, ov);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 32; ++x)
            if (r0 + x < rows) dst[(size_t)(r0 + x) * row_stride] = __float2bfloat16_rn(ov[x]);
    }
}

__global__ void __maxnreg__(128)
chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                const __grid_constant__ CUtensorMap tm_r, const TcParams p)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // Align by offsetting the shared array itself (not via an integer round trip), so
    // the compiler keeps every access below in the shared state space (LDS/STS).
    unsigned char *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + OFF_MISC + 4);
    const TcCtl ctl{bar, abort_flag};

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.x;
    const int hq = h / (p.Hv / p.Hqk);
    // This CTA's tokens, start state, final state and output (see TcParams).
    int b = blockIdx.y;
    SeqSpan sq;
    bool trans = false;                          // transition run: v = 0, S0 = I
    const float *s0_src;                         // null: zero start
    float *sf_dst;                               // null: no final state
    __nv_bfloat16 *sst_dst = nullptr;            // bf16 S^T of the final state, or null
    const CUtensorMap *out_map = &tm_o;          // output rows [., out_T, Hv, 128]
    __nv_bfloat16 *out = p.o;
    int out_T = p.T, out_t0 = 0;                 // output row = token row - out_t0
    const size_t hstate = (size_t)kHeadDim * kHeadDim;
    if (p.seg_len > 0) {
        int y = blockIdx.y, k;
        if (y < p.B * p.nseg) {
            b = y / p.nseg;
            k = y % p.nseg;
            s0_src = (k == 0 && p.S0) ? p.S0 + ((size_t)b * p.Hv + h) * hstate : nullptr;
            sf_dst = p.seg_D + (((size_t)b * p.nseg + k) * p.Hv + h) * hstate;
            if (k == 0 && p.sst) sst_dst = p.sst + ((size_t)b * p.Hv + h) * hstate;
        } else {
            y -= p.B * p.nseg;
            b = y / (p.nseg - 1);
            k = 1 + y % (p.nseg - 1);
            trans = true;
            s0_src = nullptr;
            sf_dst = p.seg_M + (((size_t)b * (p.nseg - 1) + k - 1) * p.Hv + h) * hstate;
            out_map = &tm_r;
            out = p.r;
            out_T = p.T - p.seg_len;
            out_t0 = p.seg_len;
        }
        sq = SeqSpan{k * p.seg_len, min(p.seg_len, p.T - k * p.seg_len), b};
    } else {
        sq = seq_span(p, b);
        s0_src = p.S0 ? p.S0 + ((size_t)b * p.Hv + h) * hstate : nullptr;
        sf_dst = p.S_final ? p.S_final + ((size_t)b * p.Hv + h) * hstate : nullptr;
    }
    const int nchunks = (sq.L + C - 1) / C;
    const uint32_t sbase = smem_u32(sm);

    if (tid == 0) {
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_v);
        prefetch_tensormap(out_map);
        for (int i = 0; i < (int)NBAR; ++i) mbar_init(&bar[i], many_arrivals(i) ? 128 : 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (trans) {   // transition run: v = 0 for every chunk, so the V tile is zero once
        for (int x = tid; x < 2 * (int)TILE / 16; x += NT)
            reinterpret_cast<uint4 *>(sm + OFF_V)[x] = make_uint4(0u, 0u, 0u, 0u);
        fence_proxy_async_smem();
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
        // K/Q (NKQ stages) and V (one buffer) are independent queues: whichever has
        // a free buffer is loaded next.
        if (lane == 0) {
            int nkq = 0, nv = 0;
            int issued_kq[NKQ] = {-1, -1, -1}, issued_v = -1;
            long long idle_since = clock64();
            while (nkq < nchunks || nv < nchunks) {
                if (*abort_flag) break;
                bool issued = false;
                if (nkq < nchunks &&
                    (nkq < NKQ || mbar_test(&bar[B_KQ_EMPTY + nkq % NKQ], ((nkq / NKQ) - 1) & 1))) {
                    const int s = nkq % NKQ, t0 = sq.tb + nkq * C;
                    unsigned char *st = sm + OFF_KQ + s * KQ_STAGE;
                    mbar_arrive_expect_tx(&bar[B_KQ_FULL + s], KQ_STAGE);
                    tma_load_4d(st + 0 * TILE, &tm_k, &bar[B_KQ_FULL + s], 0, hq, t0, sq.bt);
                    tma_load_4d(st + 1 * TILE, &tm_q, &bar[B_KQ_FULL + s], 0, hq, t0, sq.bt);
                    tma_load_4d(st + 2 * TILE, &tm_k, &bar[B_KQ_FULL + s], 64, hq, t0, sq.bt);
                    tma_load_4d(st + 3 * TILE, &tm_q, &bar[B_KQ_FULL + s], 64, hq, t0, sq.bt);
                    issued_kq[s] = nkq++;
                    issued = true;
                    // the stage's next chunk into L2, so that its load is an L2 hit
                    // (on a lightly loaded GPU: with every SM busy the extra requests
                    // cost more than the latency they hide)
                    const int cf = nkq - 1 + NKQ;
                    if (p.l2_prefetch && cf < nchunks) {
                        const int tf = sq.tb + cf * C;
                        tma_prefetch_4d(&tm_k, 0, hq, tf, sq.bt);
                        tma_prefetch_4d(&tm_q, 0, hq, tf, sq.bt);
                        tma_prefetch_4d(&tm_k, 64, hq, tf, sq.bt);
                        tma_prefetch_4d(&tm_q, 64, hq, tf, sq.bt);
                        if (!trans) {
                            tma_prefetch_4d(&tm_v, 0, h, tf, sq.bt);
                            tma_prefetch_4d(&tm_v, 64, h, tf, sq.bt);
                        }
                    }
                }
                if (nv < nchunks && (nv < 1 || mbar_test(&bar[B_V_EMPTY], (nv - 1) & 1))) {
                    if (trans) {                 // v = 0: the zero tile stays; only signal it
                        mbar_arrive(&bar[B_V_FULL]);
                    } else {
                        const int t0 = sq.tb + nv * C;
                        mbar_arrive_expect_tx(&bar[B_V_FULL], 2 * TILE);
                        tma_load_4d(sm + OFF_V, &tm_v, &bar[B_V_FULL], 0, h, t0, sq.bt);
                        tma_load_4d(sm + OFF_V + TILE, &tm_v, &bar[B_V_FULL], 64, h, t0, sq.bt);
                        issued_v = nv;
                    }
                    ++nv;
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
            if (*abort_flag) {
                // Let copies still in flight land before the CTA's memory goes away.
                for (int s = 0; s < NKQ; ++s)
                    if (issued_kq[s] >= 0)
                        mbar_wait(&bar[B_KQ_FULL + s], (issued_kq[s] / NKQ) & 1, 1ll << 28);
                if (issued_v >= 0) mbar_wait(&bar[B_V_FULL], issued_v & 1, 1ll << 28);
            }
        }
    } else if (warp == 1) {
        // ======================================================== MMA issuer
        // Issues, as soon as their inputs are ready, in this priority order:
        //   YS(c): S^T += (U^T diag(g)) K, O^T += U^T P^T   needs U^T bf16 and P of c
        //   UO(c): U^T += S^T (-W)^T, O^T = S^T Q^T   needs S^T bf16 and W of c
        //   WU(c): W^T, U~^T                          needs the solve of c and the
        //                                             UO MMAs of c-1 completed
        //   G(c):  [K;Q] K^T                          needs the K/Q tiles of c
        if (lane == 0) {
            int ng = 0, nwu = 0, nuo = 0, nys = 0;
            long long idle_since = clock64();
            while (nys < nchunks) {
                if (*abort_flag) break;
                bool issued = false;
                if (nys < nuo && mbar_test(&bar[u_ready(nys)], (nys >> 1) & 1) &&
                    mbar_test(&bar[B_PREP + (nys & 1)], (nys >> 1) & 1)) {
                    const int c = nys, s = c & 1;
                    tc_fence_after();
                    const uint32_t col_o = COL_O + s * 64;
                    // the state update first: the next chunk waits for it
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_bf16_ts(tmem + COL_S, tmem + COL_U + s * 64 + 32 + k * 8,
                                    smem_desc_sw128(sbase + OFF_KQ + (c % NKQ) * KQ_STAGE + k * 2048, 2 * TILE, 1024),
                                    ID_S, true);
                    mma_commit(&bar[B_S_FULL]);
                    mma_commit(&bar[B_KQ_EMPTY + c % NKQ]);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_bf16_ts(tmem + col_o, tmem + COL_U + s * 64 + k * 8,
                                    smem_desc_sw128(sbase + OFF_P + s * TILE + k * 32, 16, 1024), ID_O, true);
                    mma_commit(&bar[B_O_FULL + s]);
                    GDN_TRACE_AT(c, 5, true);
                    ++nys;
                    issued = true;
                } else if (nuo < nwu && mbar_test(&bar[B_S_READY], nuo & 1) &&
                           (nuo < 2 || mbar_test(&bar[B_O_FREE + (nuo & 1)], ((nuo >> 1) - 1) & 1))) {
                    const int c = nuo, s = c & 1;
                    const uint32_t st = sbase + OFF_KQ + (c % NKQ) * KQ_STAGE;
                    const uint32_t col_o = COL_O + s * 64, col_u = COL_U + s * 64;
                    tc_fence_after();
                    GDN_TRACE_AT(c, 1, true);
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        mma_bf16_ts(tmem + col_u, tmem + COL_W + k * 8,
                                    smem_desc_sw128(sbase + OFF_W + k * 2048, 2 * TILE, 1024), ID_U, true);
                    mma_commit(&bar[B_U_FULL]);
                    // S-part of O with Q~ = diag(gamma) Q (scaled in place by the prep)
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint32_t koff = (k >> 2) * 2 * TILE + (k & 3) * 32;
                        mma_bf16_ts(tmem + col_o, tmem + COL_W + k * 8,
                                    smem_desc_sw128(st + TILE + koff, 16, 1024), ID_O, k > 0);
                    }
                    mma_commit(&bar[B_X_FULL]);
                    GDN_TRACE_AT(c, 2, true);
                    ++nuo;
                    issued = true;
                } else if (nwu < ng && mbar_test(&bar[B_SOLVE + (nwu & 1)], (nwu >> 1) & 1) &&
                           mbar_test(&bar[B_V_FULL], nwu & 1) &&
                           // the UO MMAs of c-1 (last readers of the S^T bf16 in the W^T
                           // columns) have completed; so have the YS MMAs of c-2 (readers
                           // of the U^T bf16 in this U^T buffer), issued before them
                           (nwu < 1 || mbar_test(&bar[B_X_FULL], (nwu - 1) & 1))) {
                    const int c = nwu, s = c & 1;
                    const uint32_t st = sbase + OFF_KQ + (c % NKQ) * KQ_STAGE;
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
                    mma_commit(&bar[B_W_FULL + s]);
                    mma_commit(&bar[B_V_EMPTY]);
                    GDN_TRACE_AT(c, 6, true);
                    ++nwu;
                    issued = true;
                } else if (ng < nchunks && mbar_test(&bar[B_KQ_FULL + ng % NKQ], (ng / NKQ) & 1) &&
                           (ng < 1 || mbar_test(&bar[B_G_FREE], (ng - 1) & 1))) {
                    const int c = ng;
                    const uint32_t st = sbase + OFF_KQ + (c % NKQ) * KQ_STAGE;
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint32_t koff = (k >> 2) * 2 * TILE + (k & 3) * 32;
                        mma_bf16(tmem + COL_G, smem_desc_sw128(st + koff, 16, 1024),
                                 smem_desc_sw128(st + koff, 16, 1024), ID_G, k > 0);
                    }
                    mma_commit(&bar[B_G_FULL + (c & 1)]);
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
    } else if (warp < 10) {
        // ======================================================== prep warpgroups
        // Two warpgroups prepare alternate chunks (warps 2-5 the even ones, warps
        // 6-9 the odd ones), each with its own A / solve scratch and P buffer; Bw
        // and Bu are shared and written in chunk order (each writer waits for the
        // MMAs of the chunk before that read them).
        const int wg = (warp - 2) >> 2;               // 0: even chunks, 1: odd chunks
        const int pt = tid - 64 - 128 * wg;           // 0..127
        const int nb = wg ? 3 : 1;                    // named barrier of this warpgroup
        const int q4 = warp & 3;                      // TMEM lane quarter
        const int row = q4 * 32 + lane;               // TMEM lane = matrix row
        const uint32_t t_row = tmem + ((uint32_t)(q4 * 32) << 16);
        float *sA = reinterpret_cast<float *>(sm + OFF_A + wg * SA_BYTES);
        float *sY = reinterpret_cast<float *>(sm + OFF_Y + wg * SY_BYTES);
        const bool gate_warp = pt < 32;               // first warp of the warpgroup
        bool ok = true;
        // gate prefetch: alpha, beta of this warpgroup's next chunk are in flight
        // while the current one is prepared
        float nx_a0 = 1.f, nx_a1 = 1.f, nx_b0 = 0.f, nx_b1 = 0.f;
        if (gate_warp && wg < nchunks) load_gates(p, sq, h, wg, lane, nx_a0, nx_a1, nx_b0, nx_b1);
        for (int c = wg; c < nchunks && ok; c += 2) {
            const int s = c & 1, gb = c % NGATE;
            float *gv = reinterpret_cast<float *>(sm + OFF_GATE + gb * GATE_BUF);
            GDN_TRACE_AT(c, 8, pt == 0);
            // ---- gates (first warp): b in log2 units, gamma, beta, g, beta gamma, e32;
            //      padded rows carry alpha = 1, beta = 0 (neutral).  The chain is done
            //      with the gates of chunk c - NGATE, the last user of this buffer.
            if (c >= NGATE) ok = ctl.wait(B_GFREE + gb, ((c / NGATE) - 1) & 1);
            if (ok && gate_warp) {
                const float a0 = nx_a0, a1 = nx_a1, be0 = nx_b0, be1 = nx_b1;
                if (c + 2 < nchunks) load_gates(p, sq, h, c + 2, lane, nx_a0, nx_a1, nx_b0, nx_b1);
                compute_gates(gv, a0, a1, be0, be1, lane);
            }
            ok = named_and(nb, 128, ok);
            if (!ok) break;
            if (pt == 0) mbar_arrive(&bar[B_GATES + gb]);
            GDN_TRACE_AT(c, 9, pt == 0);
            // ---- grams -> A rows (lanes 0-63, fp32 into sA) and P rows (lanes 64-127,
            //      bf16 pairs kept in registers until the P buffer is free).  Decay
            //      factors Gam[r][x] = prod_{x<j<=r} alpha_j are running products along
            //      the row (no special-function work).
            ok = ctl.wait(B_KQ_FULL + c % NKQ, (c / NKQ) & 1) && ctl.wait(B_G_FULL + s, (c >> 1) & 1);
            ok = named_and(nb, 128, ok);
            if (!ok) break;
            tc_fence_after();
            GDN_TRACE_AT(c, 10, pt == 0);
            uint32_t pk[32];
            {
                float g0[32], g1[32];
                tmem_ld32(t_row + COL_G, g0);
                tmem_ld32(t_row + COL_G + 32, g1);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(&bar[B_G_FREE]);
                ap_row_values(gv, row, g0, g1);
                if (row < 64) {
                    float4 *dst = reinterpret_cast<float4 *>(sA + row * LDA);
#pragma unroll
                    for (int x = 0; x < 8; ++x)
                        dst[x] = make_float4(g0[4 * x], g0[4 * x + 1], g0[4 * x + 2], g0[4 * x + 3]);
#pragma unroll
                    for (int x = 0; x < 8; ++x)
                        dst[8 + x] = make_float4(g1[4 * x], g1[4 * x + 1], g1[4 * x + 2], g1[4 * x + 3]);
                }
#pragma unroll
                for (int x = 0; x < 16; ++x) {
                    pk[x] = pack_bf16x2(g0[2 * x], g0[2 * x + 1]);
                    pk[16 + x] = pack_bf16x2(g1[2 * x], g1[2 * x + 1]);
                }
            }
            named_sync(nb, 128);
            GDN_TRACE_AT(c, 11, pt == 0);
            // ---- T = (I + A)^-1, then Bw = T diag(beta gamma) (threads 0-63, row pt)
            //      and Bu = T diag(beta) (threads 64-127, row pt - 64) as bf16 operands
            unit_lower_inverse(sA, sY, pt, nb);
            GDN_TRACE_AT(c, 22, pt == 0);
            // the shared Bw, Bu were last read by the W^T / U~^T MMAs of c-1
            ok = named_and(nb, 128, c < 1 || ctl.wait(B_W_FULL + ((c - 1) & 1), ((c - 1) >> 1) & 1));
            if (!ok) break;
            GDN_TRACE_AT(c, 23, pt == 0);
            write_bw_bu(gv, sA, pt, sm + OFF_BW, sm + OFF_BU);
            // ---- Q~ = diag(gamma) Q in place (row pt >> 1, key half pt & 1): the grams
            //      have read Q; the UO MMAs, issued after SOLVE, read Q~
            {
                const int i = pt >> 1, half = pt & 1;
                unsigned char *qt = sm + OFF_KQ + (c % NKQ) * KQ_STAGE + (2 * half + 1) * TILE;
                scale_row_bf16(qt, qt, i, gv[GV_GAM + i]);
            }
            fence_proxy_async_smem();
            mbar_arrive(&bar[B_SOLVE + s]);
            GDN_TRACE_AT(c, 12, pt == 0);
            // ---- P into this parity's buffer, last read by the YS MMAs of c-2
            ok = named_and(nb, 128, c < 2 || ctl.wait(B_O_FULL + s, ((c - 2) >> 1) & 1));
            if (!ok) break;
            tc_fence_after();
            GDN_TRACE_AT(c, 13, pt == 0);
            if (row >= 64) {
                unsigned char *ptile = sm + OFF_P + s * TILE;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch)
                    *reinterpret_cast<uint4 *>(ptile + sw128_chunk(row - 64, ch)) =
                        make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bar[B_PREP + s]);
            GDN_TRACE_AT(c, 14, pt == 0);
        }
    } else {
        // ======================================================== chain warpgroup
        const int q4 = warp & 3;
        const int j = q4 * 32 + lane;                 // TMEM lane = value column j (W^T: key dim d)
        const uint32_t t_row = tmem + ((uint32_t)(q4 * 32) << 16);
        const bool leader = (j == 0);
        bool ok = true;
        // initial state: S^T[j][d] = S0[d][j]
        {
            const float *src = s0_src;
#pragma unroll 1
            for (int c0 = 0; c0 < kHeadDim; c0 += 32) {
                float v[32];
#pragma unroll
                for (int x = 0; x < 32; ++x)
                    v[x] = trans ? (c0 + x == j ? 1.f : 0.f) : src ? src[(size_t)(c0 + x) * kHeadDim + j] : 0.f;
                tmem_st32(t_row + COL_S + c0, v);
            }
            tmem_wait_st();
        }
        // O epilogue of chunk cp: O^T (lane j) -> bf16 o[t][h][j].  A full chunk is
        // staged as a bf16 tile [r][j] in the W tile (idle from the end of the UO
        // MMAs of the chunk after cp to the next W conversion, which first waits
        // for the store to have read it) and written by one TMA store; a chunk cut
        // by the end of its sequence is stored row by row from registers (a warp
        // writes 64 contiguous bytes per row), rows past the end skipped.
        const size_t row_stride = (size_t)p.Hv * kHeadDim;
        __nv_bfloat16 *out_h = out + ((size_t)sq.bt * out_T + (sq.tb - out_t0)) * row_stride +
                               (size_t)h * kHeadDim + j;
        auto epilogue = [&](int cp) -> bool {
            if (leader) bulk_wait_group_read0();     // the previous store has read the W tile
            if (!named_and(2, 128, ctl.wait(B_O_FULL + (cp & 1), (cp >> 1) & 1))) return false;
            tc_fence_after();
            const uint32_t col_o = COL_O + (cp & 1) * 64;
            const int rows = min(C, sq.L - cp * C);
            if (rows == C) {
                // 8 x 8 blocks (8 lanes j x 8 columns r) come out of TMEM in the m16n8
                // fragment layout and go to the [r][j] tile transposed by stmatrix
                const uint32_t stage = smem_u32(sm + OFF_W);
                const int mt = lane >> 3, mi = lane & 7;   // stored row mi of matrix mt
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
                        const int orow = 32 * cb + 8 * k + mi;          // output row r
                        const int jst = q4 * 32 + 16 * sl + 8 * g;      // first j of the block
                        stmatrix_x4_trans(stage + (jst >> 6) * TILE + sw128_chunk(orow, (jst & 63) >> 3),
                                          m[0], m[1], m[2], m[3]);
                    }
                };
#pragma unroll 1
                for (int sl = 0; sl < 2; ++sl) {             // 16-lane slab
                    uint32_t ra[16], rb[16];                 // 32-column blocks 0, 1
                    const uint32_t ta = tmem + ((uint32_t)(q4 * 32 + 16 * sl) << 16) + col_o;
                    tmem_ld16x256b_x4(ta, ra);
                    tmem_ld16x256b_x4(ta + 32, rb);
                    tmem_wait_ld();
                    emit(ra, sl, 0);
                    emit(rb, sl, 1);
                }
                tc_fence_before();
                mbar_arrive(&bar[B_O_FREE + (cp & 1)]);
                fence_proxy_async_smem();
                named_sync(2, 128);
                if (leader) {
                    tma_store_4d(out_map, sm + OFF_W, 0, h, sq.tb + cp * C - out_t0, sq.bt);
                    tma_store_4d(out_map, sm + OFF_W + TILE, 64, h, sq.tb + cp * C - out_t0, sq.bt);
                    bulk_commit_group();
                }
                return true;
            }
            tc_store_o_rows(out_h + (size_t)cp * C * row_stride, t_row + col_o, rows, row_stride);
            tc_fence_before();
            mbar_arrive(&bar[B_O_FREE + (cp & 1)]);
            return true;
        };
        for (int c = 0; c < nchunks && ok; ++c) {
            const int s = c & 1, gb = c % NGATE;
            const float *gv = reinterpret_cast<const float *>(sm + OFF_GATE + gb * GATE_BUF);
            GDN_TRACE_AT(c, 16, leader);
            // W^T (TMEM, lane d) -> W [d][r] bf16 (MN-major B of the U MMAs).  The UO
            // MMAs of c-1 have completed (X_FULL(c-1), waited in c-1) and the O
            // store staged in the W tile has read it (waited for by the leader).
            if (leader) bulk_wait_group_read0();
            ok = named_and(2, 128, ctl.wait(B_W_FULL + s, (c >> 1) & 1));
            if (!ok) break;
            tc_fence_after();
            {
                float w0[32], w1[32];
                tmem_ld32(t_row + COL_W, w0);
                tmem_ld32(t_row + COL_W + 32, w1);
                tmem_wait_ld();
                store_half_row_bf16(sm + OFF_W, j, 0, w0);
                store_half_row_bf16(sm + OFF_W, j, 1, w1);
            }
            GDN_TRACE_AT(c, 25, leader);
            // S^T -> packed bf16 A operand in the (now read) W^T columns, and
            // S^T <- gamma_{C-1} S^T
            if (c > 0) ok = ctl.wait(B_S_FULL, (c - 1) & 1);
            ok = ok && ctl.wait(B_GATES + gb, (c / NGATE) & 1);
            ok = named_and(2, 128, ok);
            if (!ok) break;
            tc_fence_after();
            GDN_TRACE_AT(c, 17, leader);
            const float glast = gv[GV_GAM + C - 1];
#pragma unroll 1
            for (int c0 = 0; c0 < kHeadDim; c0 += 64) {
                float v[64];
                uint32_t pk[32];
                tmem_ld32(t_row + COL_S + c0, v);
                tmem_ld32(t_row + COL_S + c0 + 32, v + 32);
                tmem_wait_ld();
#pragma unroll
                for (int x = 0; x < 32; ++x) pk[x] = pack_bf16x2(v[2 * x], v[2 * x + 1]);
                tmem_st32u(t_row + COL_W + (c0 >> 1), pk);
#pragma unroll
                for (int x = 0; x < 64; ++x) v[x] *= glast;
                tmem_st32(t_row + COL_S + c0, v);
                tmem_st32(t_row + COL_S + c0 + 32, v + 32);
            }
            tmem_wait_st();
            fence_proxy_async_smem();                // the W tile, for the tensor core
            tc_fence_before();
            mbar_arrive(&bar[B_S_READY]);
            GDN_TRACE_AT(c, 18, leader);
            // U^T -> packed bf16 A operands, in place: U^T (columns 0-31 of its buffer)
            // for the O update, U^T diag(g) (columns 32-63) for the state update
            ok = named_and(2, 128, ctl.wait(B_U_FULL, c & 1));
            if (!ok) break;
            tc_fence_after();
            GDN_TRACE_AT(c, 20, leader);
            {
                float u[64];
                uint32_t pk[32];
                tmem_ld32(t_row + COL_U + s * 64, u);
                tmem_ld32(t_row + COL_U + s * 64 + 32, u + 32);
                tmem_wait_ld();
#pragma unroll
                for (int x = 0; x < 32; ++x) pk[x] = pack_bf16x2(u[2 * x], u[2 * x + 1]);
                tmem_st32u(t_row + COL_U + s * 64, pk);
                const float4 *g4 = reinterpret_cast<const float4 *>(gv + GV_G);
#pragma unroll
                for (int x = 0; x < 16; ++x) {
                    const float4 g = g4[x];
                    pk[2 * x] = pack_bf16x2(u[4 * x] * g.x, u[4 * x + 1] * g.y);
                    pk[2 * x + 1] = pack_bf16x2(u[4 * x + 2] * g.z, u[4 * x + 3] * g.w);
                }
                tmem_st32u(t_row + COL_U + s * 64 + 32, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bar[u_ready(c)]);
            mbar_arrive(&bar[B_GFREE + gb]);         // gates of c no longer read
            GDN_TRACE_AT(c, 21, leader);
            // O epilogue of the previous chunk, while the YS MMAs of c run
            if (c > 0 && !(ok = epilogue(c - 1))) break;
            GDN_TRACE_AT(c, 19, leader);
        }
        if (ok && nchunks > 0) ok = epilogue(nchunks - 1);
        if (ok && sf_dst) {
            float *dst = sf_dst;
#pragma unroll 1
            for (int c0 = 0; c0 < kHeadDim; c0 += 32) {
                float v[32];
                tmem_ld32(t_row + COL_S + c0, v);
                tmem_wait_ld();
#pragma unroll
                for (int x = 0; x < 32; ++x) dst[(size_t)(c0 + x) * kHeadDim + j] = v[x];
                if (sst_dst) {   // row j of S^T, bf16: 64 contiguous bytes
                    uint4 *row = reinterpret_cast<uint4 *>(sst_dst + (size_t)j * kHeadDim + c0);
#pragma unroll
                    for (int x = 0; x < 4; ++x)
                        row[x] = make_uint4(pack_bf16x2(v[8 * x], v[8 * x + 1]), pack_bf16x2(v[8 * x + 2], v[8 * x + 3]),
                                            pack_bf16x2(v[8 * x + 4], v[8 * x + 5]), pack_bf16x2(v[8 * x + 6], v[8 * x + 7]));
                }
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

}  // namespace

bool chunk_tc_available() { return encode_fn() != nullptr; }

cudaError_t chunk_tc_take_error(unsigned *out)
{
    unsigned v = 0, zero = 0;
    cudaError_t err = cudaMemcpyFromSymbol(&v, g_tc_error, sizeof(v));
    if (err == cudaSuccess && v) err = cudaMemcpyToSymbol(g_tc_error, &zero, sizeof(zero));
    *out = v;
    return err;
}

#ifdef GDN_TRACE
// Copies the trace of the last traced launch (kTraceChunks x kTraceSlots ns stamps).
extern "C" int gdn_trace_read(unsigned long long *host, int n)
{
    if (n < kTraceChunks * kTraceSlots) return -1;
    return (int)cudaMemcpyFromSymbol(host, g_trace, sizeof(g_trace));
}
#endif

// A grid that leaves at least half of the SMs idle.
static int light_grid(long long ctas)
{
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return 2 * ctas <= sms ? 1 : 0;
}

cudaError_t launch_chunk_tc(const ChunkArgs &a, cudaStream_t stream)
{
    CUtensorMap tk, tq, tv, to;
    const int rows_b = a.cu_seqlens ? 1 : a.B;   // batch rows of the token arrays
    if (!make_map(&tk, a.k, rows_b, a.T, a.Hqk) || !make_map(&tq, a.q, rows_b, a.T, a.Hqk) ||
        !make_map(&tv, a.v, rows_b, a.T, a.Hv) || !make_map(&to, a.o, rows_b, a.T, a.Hv))
        return cudaErrorInvalidValue;
    cudaError_t err = cudaFuncSetAttribute(chunk_tc_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)SMEM_BYTES);
    if (err != cudaSuccess) return err;
    TcParams p{a.alpha, a.beta, a.S0, a.S_final, a.T, a.Hqk, a.Hv,
               static_cast<__nv_bfloat16 *>(a.o), a.cu_seqlens};
    p.l2_prefetch = light_grid((long long)a.Hv * a.B);
    chunk_tc_kernel<<<dim3((unsigned)a.Hv, (unsigned)a.B), NT, SMEM_BYTES, stream>>>(tk, tq, tv, to, to, p);
    return cudaGetLastError();
}

cudaError_t launch_chunk_tc_segments(const ChunkArgs &a, int seg_len, int nseg, float *segD,
                                     float *segM, __nv_bfloat16 *R, __nv_bfloat16 *sst,
                                     cudaStream_t stream)
{
    CUtensorMap tk, tq, tv, to, tr;
    if (!make_map(&tk, a.k, a.B, a.T, a.Hqk) || !make_map(&tq, a.q, a.B, a.T, a.Hqk) ||
        !make_map(&tv, a.v, a.B, a.T, a.Hv) || !make_map(&to, a.o, a.B, a.T, a.Hv) ||
        !make_map(&tr, R, a.B, a.T - seg_len, a.Hv))
        return cudaErrorInvalidValue;
    cudaError_t err = cudaFuncSetAttribute(chunk_tc_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)SMEM_BYTES);
    if (err != cudaSuccess) return err;
    TcParams p{a.alpha, a.beta, a.S0, nullptr, a.T, a.Hqk, a.Hv,
               static_cast<__nv_bfloat16 *>(a.o), nullptr, a.B, seg_len, nseg, segD, segM, R, sst};
    const unsigned rows = (unsigned)(a.B * nseg + a.B * (nseg - 1));
    p.l2_prefetch = light_grid((long long)a.Hv * rows);
    chunk_tc_kernel<<<dim3((unsigned)a.Hv, rows), NT, SMEM_BYTES, stream>>>(tk, tq, tv, to, tr, p);
    return cudaGetLastError();
}

}  // namespace gdn
