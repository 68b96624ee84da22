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
//               MMAs for the block merges), Bw and Bu, and K~
//   warps 6-9   "chain" warpgroup, the state-dependent path: S^T -> bf16
//               operand (+ decay of the fp32 state), W^T -> bf16 W operand,
//               U^T -> bf16 operand, the gamma scaling of the S-part of O^T in
//               TMEM, and the O epilogue (staged in shared memory, one TMA store)
// The U^T and O^T accumulators are double-buffered, so the prep work of the
// next chunk never waits for the state-dependent chain of the current one.
//
// Every wait is bounded.  On a timeout the CTA raises a device error flag, the
// other roles see a shared abort flag and stop, in-flight copies and MMAs are
// drained (again with a bound) and TMEM is freed before returning.
#include "tc_common.cuh"

namespace gdn {

namespace {

constexpr int NT = 320;            // 10 warps

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
constexpr uint32_t OFF_Y = OFF_A + 64 * LDA * 4;  // solve scratch, fp32 [32][LDY]
constexpr uint32_t OFF_GATE = OFF_Y + 32 * LDY * 4;  // 2 buffers of gate vectors
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
    B_PREP = 9,      // prep: K~ written, the K of its stage read (128)
    B_GATES = 10,    // 2: gates of a chunk written
    B_S_READY = 12,  // chain: S^T and W bf16 written, W^T read from TMEM (128)
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

__global__ void __launch_bounds__(NT, 1)
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
    const Ctl ctl{bar, abort_flag};

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.x;
    const int hq = h / (p.Hv / p.Hqk);
    // This CTA's tokens, start state, final state and output (see TcParams).
    int b = blockIdx.y;
    SeqSpan sq;
    bool trans = false;                          // transition run: v = 0, S0 = I
    const float *s0_src;                         // null: zero start
    float *sf_dst;                               // null: no final state
    const CUtensorMap *out_map = &tm_o;
    int out_t0 = 0;                              // output row = token row - out_t0
    const size_t hstate = (size_t)kHeadDim * kHeadDim;
    if (p.seg_len > 0) {
        int y = blockIdx.y, k;
        if (y < p.B * p.nseg) {
            b = y / p.nseg;
            k = y % p.nseg;
            s0_src = (k == 0 && p.S0) ? p.S0 + ((size_t)b * p.Hv + h) * hstate : nullptr;
            sf_dst = p.seg_D + (((size_t)b * p.nseg + k) * p.Hv + h) * hstate;
        } else {
            y -= p.B * p.nseg;
            b = y / (p.nseg - 1);
            k = 1 + y % (p.nseg - 1);
            trans = true;
            s0_src = nullptr;
            sf_dst = p.seg_M + (((size_t)b * (p.nseg - 1) + k - 1) * p.Hv + h) * hstate;
            out_map = &tm_r;
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
        for (int i = 0; i < (int)NBAR; ++i) {
            const bool many = (i == B_SOLVE || i == B_PREP || i == B_S_READY || i == B_U_READY ||
                               i == B_U_READY1 || i == B_O_FREE || i == B_O_FREE + 1 ||
                               i == B_G_FREE);
            mbar_init(&bar[i], many ? 128 : 1);
        }
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
        if (lane == 0) {
            bool ok = true;
            int issued_kq0 = -1, issued_kq1 = -1, issued_v = -1;
            for (int c = 0; c < nchunks && ok; ++c) {
                const int s = c & 1, t0 = sq.tb + c * C;
                if (c >= 2) ok = ctl.wait(B_KQ_EMPTY + s, ((c >> 1) - 1) & 1);
                if (!ok) break;
                unsigned char *st = sm + OFF_KQ + s * KQ_STAGE;
                mbar_arrive_expect_tx(&bar[B_KQ_FULL + s], KQ_STAGE);
                tma_load_4d(st + 0 * TILE, &tm_k, &bar[B_KQ_FULL + s], 0, hq, t0, sq.bt);
                tma_load_4d(st + 1 * TILE, &tm_q, &bar[B_KQ_FULL + s], 0, hq, t0, sq.bt);
                tma_load_4d(st + 2 * TILE, &tm_k, &bar[B_KQ_FULL + s], 64, hq, t0, sq.bt);
                tma_load_4d(st + 3 * TILE, &tm_q, &bar[B_KQ_FULL + s], 64, hq, t0, sq.bt);
                if (s) issued_kq1 = c; else issued_kq0 = c;
                if (c >= 1) ok = ctl.wait(B_V_EMPTY, (c - 1) & 1);
                if (!ok) break;
                if (trans) {                 // v = 0: the zero tile stays; only signal it
                    mbar_arrive(&bar[B_V_FULL]);
                    continue;
                }
                mbar_arrive_expect_tx(&bar[B_V_FULL], 2 * TILE);
                tma_load_4d(sm + OFF_V, &tm_v, &bar[B_V_FULL], 0, h, t0, sq.bt);
                tma_load_4d(sm + OFF_V + TILE, &tm_v, &bar[B_V_FULL], 64, h, t0, sq.bt);
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
                           (nwu < 1 || mbar_test(&bar[B_S_READY], (nwu - 1) & 1)) &&
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
        if (warp == 2 && nchunks > 0) load_gates(p, sq, h, 0, lane, nx_a0, nx_a1, nx_b0, nx_b1);
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
                const float a0 = nx_a0, a1 = nx_a1, be0 = nx_b0, be1 = nx_b1;
                if (c + 1 < nchunks) load_gates(p, sq, h, c + 1, lane, nx_a0, nx_a1, nx_b0, nx_b1);
                compute_gates(gv, a0, a1, be0, be1, lane);
            }
            named_sync(1, 128);
            if (pt == 0) mbar_arrive(&bar[B_GATES + s]);
            GDN_TRACE_AT(c, 9, pt == 0);
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
                float g0[32], g1[32];
                tmem_ld32(t_row + COL_G, g0);
                tmem_ld32(t_row + COL_G + 32, g1);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(&bar[B_G_FREE]);
                ap_row(gv, row, g0, g1, sA, sm + OFF_P + s * TILE);
            }
            named_sync(1, 128);
            GDN_TRACE_AT(c, 11, pt == 0);
            // ---- T = (I + A)^-1, then Bw = T diag(beta gamma) (threads 0-63, row pt)
            //      and Bu = T diag(beta) (threads 64-127, row pt - 64) as bf16 operands
            unit_lower_inverse(sA, sY, pt, 1);
            GDN_TRACE_AT(c, 22, pt == 0);
            // the single-buffered Bw, Bu were last read by the W^T / U~^T MMAs of c-1
            ok = named_and(1, 128, c < 1 || ctl.wait(B_W_FULL, (c - 1) & 1));
            if (!ok) break;
            GDN_TRACE_AT(c, 23, pt == 0);
            write_bw_bu(gv, sA, pt, sm + OFF_BW, sm + OFF_BU);
            fence_proxy_async_smem();
            mbar_arrive(&bar[B_SOLVE]);
            GDN_TRACE_AT(c, 12, pt == 0);
            // ---- K~ = diag(g) K.  The single-buffered K~ (and P of chunk c-1) must no
            //      longer be read by the previous chunk's MMAs.  (W^T -> W is the
            //      chain's: it waits for the W^T MMA of c anyway.)
            ok = named_and(1, 128, c < 1 || ctl.wait(B_O_FULL, (c - 1) & 1));
            if (!ok) break;
            tc_fence_after();
            GDN_TRACE_AT(c, 13, pt == 0);
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
        // Staged O^T of chunk cp (bf16 tile [r][j] at OFF_U) -> o: one TMA store,
        // except for the last chunk of a packed sequence that ends inside it,
        // whose rows past the end belong to the next sequence: its rows are
        // stored one by one (rows past the array's end are clipped by the TMA).
        auto store_staged_o = [&](int cp, bool wait_read) {
            const int rows = min(C, sq.L - cp * C);
            if (p.cu_seqlens && rows < C) {
                const size_t row_stride = (size_t)p.Hv * kHeadDim;
                const unsigned char *ot = sm + OFF_U + (j >> 6) * TILE;
                __nv_bfloat16 *dst = p.o + ((size_t)sq.bt * p.T + sq.tb + (size_t)cp * C) * row_stride +
                                     (size_t)h * kHeadDim + j;
#pragma unroll 1
                for (int r = 0; r < rows; ++r)
                    dst[(size_t)r * row_stride] =
                        *reinterpret_cast<const __nv_bfloat16 *>(ot + sw128_offset(r, j & 63));
            } else if (leader) {
                tma_store_4d(out_map, sm + OFF_U, 0, h, sq.tb + cp * C - out_t0, sq.bt);
                tma_store_4d(out_map, sm + OFF_U + TILE, 64, h, sq.tb + cp * C - out_t0, sq.bt);
                bulk_commit_group();
                if (wait_read) bulk_wait_group_read0();
            }
        };
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
            GDN_TRACE_AT(c, 24, leader);
            // W^T (TMEM, lane d) -> W [d][r] bf16 (MN-major B of the U MMAs); the U MMAs
            // of c-1 that read W last have completed (U_FULL(c-1) waited in c-1)
            ok = named_and(2, 128, ctl.wait(B_W_FULL, c & 1));
            if (!ok) break;
            GDN_TRACE_AT(c, 25, leader);
            tc_fence_after();
            {
                float w0[32], w1[32];
                tmem_ld32(t_row + COL_W, w0);
                tmem_ld32(t_row + COL_W + 32, w1);
                tmem_wait_ld();
                store_half_row_bf16(sm + OFF_W, j, 0, w0);
                store_half_row_bf16(sm + OFF_W, j, 1, w1);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bar[B_S_READY]);            // bf16 S^T and W written
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
                store_staged_o(cp, true);      // staging must be read before U^T reuses it
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
                store_staged_o(cp, false);
            }
        }
        if (ok && sf_dst) {
            float *dst = sf_dst;
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
    chunk_tc_kernel<<<dim3((unsigned)a.Hv, (unsigned)a.B), NT, SMEM_BYTES, stream>>>(tk, tq, tv, to, to, p);
    return cudaGetLastError();
}

cudaError_t launch_chunk_tc_segments(const ChunkArgs &a, int seg_len, int nseg, float *segD,
                                     float *segM, __nv_bfloat16 *R, cudaStream_t stream)
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
               static_cast<__nv_bfloat16 *>(a.o), nullptr, a.B, seg_len, nseg, segD, segM};
    const unsigned rows = (unsigned)(a.B * nseg + a.B * (nseg - 1));
    chunk_tc_kernel<<<dim3((unsigned)a.Hv, rows), NT, SMEM_BYTES, stream>>>(tk, tq, tv, to, tr, p);
    return cudaGetLastError();
}

}  // namespace gdn
