// Chunkwise (WY) prefill on tcgen05 for few (sequence, V head) pairs: a cluster of
// two CTAs per pair.  Same mathematics, operand values and rounding points as
// gdn_chunk_tc.cu ("Qwen3.8-Flash-Next 技术总结 -- Qwen4 架构的探路者", section 2.1
// "Gated DeltaNet"; the chunk equations are in that file's header).
//
// With one CTA per pair a B=1 prefill of 48 V heads leaves 100 of 148 SMs idle,
// and each CTA is bound by the CUDA-core work that prepares a chunk (grams ->
// A, P -> triangular inverse), not by the state-dependent chain.  Here the
// S-independent preparation moves to a helper CTA with two prep warpgroups that
// take alternate chunks, and the main CTA keeps the chain:
//
//   rank 1, helper   warp 0: TMA of K, Q into a 3-stage ring; warp 1: grams
//                    [K;Q] K^T; warps 2-5 / 6-9: prep of even / odd chunks -- gates,
//                    A and P, T = (I + A)^-1 -- then two bulk copies (shared::cta ->
//                    shared::cluster, no multicast) into the main CTA's receive slot
//                    of the chunk (three slots, chunk c in slot c % 3): one bf16 tile
//                    packing Bu = T diag(beta) (lower triangle) with Bw^T =
//                    (T diag(beta gamma))^T (strict upper), the P tile, and the
//                    gamma, g and beta gamma vectors -- 16.75 KB a chunk, because
//                    the SM-to-SM path is far slower than shared memory
//   rank 0, main     warp 0: TMA of Q, V; warp 1: MMA issuer; warps 2-5: the state
//                    chain; warps 6-9 work on the slots around it: split the packed
//                    tile into Bu and Bw^T, turn W^T from the tensor cores into a
//                    bf16 W tile (over the dead Bu and Bw^T), scale K -> K~ =
//                    diag(g) K in place, and, once a chunk's MMAs have completed,
//                    release its slot (TMA of the K of the chunk three ahead into
//                    it, remote arrive to the helper) and store its O from
//                    registers
//
// The chain signals the state update as soon as the bf16 U^T operand is written,
// ahead of the gamma scaling of O, so its loop is S -> bf16 S -> U MMAs -> bf16
// U -> state MMAs.  Every wait is bounded; every CTA reaches the final cluster
// barrier, so no CTA exits while its peer may still access its memory.
#include "tc_common.cuh"

namespace gdn {
namespace {

constexpr int NT = 320;            // 10 warps in both CTAs
constexpr int CLUSTER = 2;
constexpr int NSTAGE = 3;          // helper K/Q ring
constexpr int NSLOT = 3;           // receive slots of the main CTA: chunk c uses slot c % 3

// ---- receive slot (main CTA)
constexpr uint32_t SL_K = 0;                  // K [r][d] (2 tiles) -> K~ in place
constexpr uint32_t SL_X = 2 * TILE;           // packed Bu / Bw^T -> Bu [r][i] in place
constexpr uint32_t SL_BWT = 3 * TILE;         // Bw^T [i][r] (MN-major B of W^T = K^T Bw^T)
constexpr uint32_t SL_W = SL_X;               // W [d][r] bf16 over Bu and Bw^T once both are read
constexpr uint32_t SL_P = 4 * TILE;           // P [r][i]
constexpr uint32_t SL_VEC = 5 * TILE;         // gamma_r, g_i, beta_i gamma_i: 3 x 64 floats
constexpr uint32_t VEC_BYTES = 3 * 64 * 4;
constexpr uint32_t SLOT = 5 * TILE + 1024;
constexpr uint32_t SEND_X = TILE;                  // bulk copy 1: packed tile -> SL_X
constexpr uint32_t SEND_PV = TILE + VEC_BYTES;     // bulk copy 2: [P vectors] -> SL_P
constexpr uint32_t K_BYTES = 2 * TILE;             // K tiles, loaded by the main CTA's slot warpgroup

// ---- main CTA shared memory
constexpr uint32_t Q_STAGE = 2 * TILE;        // [Q d0-63][Q d64-127]
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_V = OFF_Q + 2 * Q_STAGE;
constexpr uint32_t OFF_SLOT = OFF_V + 2 * TILE;
constexpr uint32_t OFF_S = OFF_SLOT + NSLOT * SLOT;   // S^T bf16 [j][d]
constexpr uint32_t OFF_U = OFF_S + 4 * TILE;          // U^T bf16 [j][i]
constexpr uint32_t MAIN_END = OFF_U + 2 * TILE;

// ---- helper CTA shared memory
constexpr uint32_t KQ_STAGE = 4 * TILE;       // [K d0-63][Q d0-63][K d64-127][Q d64-127]
constexpr uint32_t H_OFF_KQ = 0;
constexpr uint32_t WG_X = 0;                             // per prep warpgroup: packed tile,
constexpr uint32_t WG_P = TILE;                          // then P and the vectors (contiguous)
constexpr uint32_t WG_A = 2 * TILE + 1024;               // fp32 A / T
constexpr uint32_t WG_Y = WG_A + 64 * LDA * 4;           // solve scratch
constexpr uint32_t WG_GATE = WG_Y + 32 * LDY * 4;        // gate vectors
constexpr uint32_t WG_BYTES = (WG_GATE + GATE_BUF + 1023) / 1024 * 1024;
constexpr uint32_t H_OFF_WG = H_OFF_KQ + NSTAGE * KQ_STAGE;
constexpr uint32_t HELP_END = H_OFF_WG + 2 * WG_BYTES;

constexpr uint32_t OFF_BAR = ((MAIN_END > HELP_END ? MAIN_END : HELP_END) + 7) / 8 * 8;
constexpr uint32_t NBAR = 32;
constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 16 + 1024;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory plan exceeds 227 KB");
static_assert(SEND_PV % 16 == 0 && SLOT % 1024 == 0 && WG_BYTES % 1024 == 0 && SL_P == SL_X + 2 * TILE,
              "bulk copies move 16-byte multiples between 1024-aligned tiles");

// TMEM columns
constexpr uint32_t COL_S = 0, COL_U = 128, COL_O = 256, COL_W = 384;   // main (2 U, 2 O, 2 W buffers)
constexpr uint32_t MAIN_TMEM = 512;
constexpr uint32_t HELP_TMEM = 128;                                     // helper: G of each prep WG

// W^T = K^T Bw^T with both operands MN-major
constexpr uint32_t ID_WT = idesc_bf16(128, 64, true, true);

enum : int {
    // main CTA (count 1 unless noted)
    B_Q_FULL = 0,      // 2
    B_Q_EMPTY = 2,     // 2
    B_V_FULL = 4, B_V_EMPTY = 5,
    B_RECV = 9,        // 3 (2 arrivals), per slot: K (own TMA) and the helper's bytes landed
                       // (6-8 unused)
    B_BW_READY = 12,   // 3 (128), per slot: Bu and Bw^T split out
    B_W_FULL = 15,     // W^T and U~^T MMAs done (Bu, Bw^T read)
    B_FIN = 16,        // 3 (128), per slot: W and K~ written
    B_S_READY = 19,    // (128) bf16 S^T written
    B_U_FULL = 20,
    B_UB = 21,         // 2 (128), per U^T buffer: bf16 U^T written, TMEM buffer read
    B_S_FULL = 23, B_X_FULL = 24,
    B_O_READY = 25,    // 2 (128), per O^T buffer: gamma scaling of its S-part done
    B_O_FULL = 27,     // 2, per O^T buffer
    B_O_FREE = 29,     // 2 (128), per O^T buffer: read out
    B_DRAIN = 31,
    // helper CTA
    B_KQ_FULL = 0,     // 3
    B_KQ_EMPTY = 3,    // 3
    B_G_FULL = 6,      // 2, per prep WG
    B_G_FREE = 8,      // 2 (128)
    B_SLOT_FREE = 10,  // 3, per slot of the main CTA (remote arrive by the main CTA)
    B_H_DRAIN = 13,
};

__device__ __forceinline__ uint32_t arrivals(bool main_cta, int i) {
    if (main_cta) {
        if (i >= B_RECV && i < B_RECV + NSLOT) return 2;
        const bool many = (i >= B_BW_READY && i < B_BW_READY + NSLOT) || (i >= B_FIN && i < B_FIN + NSLOT) ||
                          i == B_S_READY || i == B_UB || i == B_UB + 1 || i == B_O_READY ||
                          i == B_O_READY + 1 || i == B_O_FREE || i == B_O_FREE + 1;
        return many ? 128 : 1;
    }
    return (i == B_G_FREE || i == B_G_FREE + 1) ? 128 : 1;
}

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
__device__ __forceinline__ void remote_arrive(uint32_t rbar) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(rbar) : "memory");
}
__device__ __forceinline__ void remote_arrive_expect_tx(uint32_t rbar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cluster.shared::cluster.b64 _, [%0], %1;"
                 ::"r"(rbar), "r"(bytes) : "memory");
}
// Bulk copy of local shared memory into the peer CTA's shared memory (no
// multicast); completes `bytes` of the transaction count of the peer's mbarrier.
__device__ __forceinline__ void bulk_copy_to_peer(uint32_t rdst, uint32_t src, uint32_t bytes,
                                                  uint32_t rbar) {
    asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes"
                 " [%0], [%1], %2, [%3];"
                 ::"r"(rdst), "r"(src), "r"(bytes), "r"(rbar) : "memory");
}

// Packed tile, row r (thread pt: row pt & 63, columns 32 (pt >> 6) ...): entry
// (r, c) is Bu[r][c] = T[r][c] beta_c for c <= r and Bw[c][r] = T[c][r] beta_r
// gamma_r for c > r -- the products and roundings of the unpacked tiles.
__device__ __forceinline__ void write_packed_bu_bwt(const float *gv, const float *sA, int pt,
                                                    unsigned char *x) {
    const int r = pt & 63, hf = pt >> 6;
    const float bg_r = gv[GV_BG + r];
    float v[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        const int c = 32 * hf + e;
        v[e] = c <= r ? sA[r * LDA + c] * gv[GV_BETA + c] : sA[c * LDA + r] * bg_r;
    }
    store_half_row_bf16(x, r, hf, v);
}

// Splits the packed tile: Bu in place (upper triangle zeroed), Bw^T into its own
// tile (lower triangle zero, diagonal beta_r gamma_r -- T has a unit diagonal).
// Thread pt owns chunks 4 (pt >> 6) .. +3 of row pt & 63 in both tiles.
__device__ __forceinline__ void unpack_bu_bwt(unsigned char *x, unsigned char *bwt, const float *bg,
                                              int pt) {
    const int r = pt & 63, ch0 = 4 * (pt >> 6);
    const uint32_t diag = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(bg[r]));
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int ch = ch0 + k;
        const uint32_t off = sw128_chunk(r, ch);
        const uint4 v = *reinterpret_cast<const uint4 *>(x + off);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t bu[4], bt[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int c0 = 8 * ch + 2 * q;         // elements c0 (low half), c0 + 1 (high half)
            const uint32_t keep = (c0 <= r ? 0x0000ffffu : 0u) | (c0 + 1 <= r ? 0xffff0000u : 0u);
            bu[q] = w[q] & keep;
            bt[q] = (w[q] & ~keep) | (c0 == r ? diag : 0u) | (c0 + 1 == r ? diag << 16 : 0u);
        }
        *reinterpret_cast<uint4 *>(x + off) = make_uint4(bu[0], bu[1], bu[2], bu[3]);
        *reinterpret_cast<uint4 *>(bwt + off) = make_uint4(bt[0], bt[1], bt[2], bt[3]);
    }
}

__global__ void __launch_bounds__(NT, 1)
chunk_tc_cluster_kernel(const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_v, const TcParams p)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + OFF_MISC + 4);
    const Ctl ctl{bar, abort_flag};

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_rank();
    const int h = blockIdx.x / CLUSTER, b = blockIdx.y;
    const int hq = h / (p.Hv / p.Hqk);
    const SeqSpan sq = seq_span(p, b);           // this sequence's token rows
    const int nchunks = (sq.L + C - 1) / C;
    const uint32_t sbase = smem_u32(sm);
    const bool is_main = (rank == 0);
    const uint32_t tmem_cols = is_main ? MAIN_TMEM : HELP_TMEM;

    if (tid == 0) {
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_q);
        if (is_main) prefetch_tensormap(&tm_v);
        for (int i = 0; i < (int)NBAR; ++i) mbar_init(&bar[i], arrivals(is_main, i));
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();          // both CTAs' barriers exist before any remote access
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (is_main) {
        // ================================================================ main CTA
        if (warp == 0) {
            // ---------------------------------------------------- TMA: Q (2 stages), V
            if (lane == 0) {
                bool ok = true;
                int issued_q0 = -1, issued_q1 = -1, issued_v = -1;
                for (int c = 0; c < nchunks && ok; ++c) {
                    const int s = c & 1, t0 = sq.tb + c * C;
                    if (c >= 2) ok = ctl.wait(B_Q_EMPTY + s, ((c >> 1) - 1) & 1);
                    if (!ok) break;
                    unsigned char *qd = sm + OFF_Q + s * Q_STAGE;
                    mbar_arrive_expect_tx(&bar[B_Q_FULL + s], Q_STAGE);
                    tma_load_4d(qd, &tm_q, &bar[B_Q_FULL + s], 0, hq, t0, sq.bt);
                    tma_load_4d(qd + TILE, &tm_q, &bar[B_Q_FULL + s], 64, hq, t0, sq.bt);
                    if (s) issued_q1 = c; else issued_q0 = c;
                    if (c >= 1) ok = ctl.wait(B_V_EMPTY, (c - 1) & 1);
                    if (!ok) break;
                    mbar_arrive_expect_tx(&bar[B_V_FULL], 2 * TILE);
                    tma_load_4d(sm + OFF_V, &tm_v, &bar[B_V_FULL], 0, h, t0, sq.bt);
                    tma_load_4d(sm + OFF_V + TILE, &tm_v, &bar[B_V_FULL], 64, h, t0, sq.bt);
                    issued_v = c;
                }
                if (*abort_flag) {
                    // Let copies still in flight land before the CTA's memory goes away.
                    if (issued_q0 >= 0) mbar_wait(&bar[B_Q_FULL], (issued_q0 >> 1) & 1, 1ll << 28);
                    if (issued_q1 >= 0) mbar_wait(&bar[B_Q_FULL + 1], (issued_q1 >> 1) & 1, 1ll << 28);
                    if (issued_v >= 0) mbar_wait(&bar[B_V_FULL], issued_v & 1, 1ll << 28);
                }
            }
        } else if (warp == 1) {
            // ---------------------------------------------------- MMA issuer
            // Issues, as soon as their inputs are ready, in this priority order:
            //   YS(c): S^T += U^T K~                         needs bf16 U^T of chunk c
            //   UO(c): U^T += S^T (-W)^T, O^T = S^T Q^T      needs bf16 S^T and W of c
            //   WU(c): W^T = K^T Bw^T, U~^T = V^T Bu^T        needs Bu, Bw^T of c
            //   YO(c): O^T += U^T P^T                        needs the scaled S-part of O^T
            // W^T and U^T have two TMEM buffers each, by chunk parity.
            if (lane == 0) {
                int nwu = 0, nuo = 0, nys = 0, nyo = 0;
                long long idle_since = clock64();
                while (nyo < nchunks) {
                    if (*abort_flag) break;
                    bool issued = false;
                    if (nys < nuo && mbar_test(&bar[B_UB + (nys & 1)], (nys >> 1) & 1)) {
                        const int c = nys;
                        const uint32_t slot = sbase + OFF_SLOT + (c % NSLOT) * SLOT;
                        tc_fence_after();
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            mma_bf16(tmem + COL_S, smem_desc_sw128(sbase + OFF_U + k * 32, 16, 1024),
                                     smem_desc_sw128(slot + SL_K + k * 2048, TILE, 1024), ID_S, true);
                        mma_commit(&bar[B_S_FULL]);
                        GDN_TRACE_CL(c, 2, true);
                        ++nys;
                        issued = true;
                    } else if (nuo < nwu && mbar_test(&bar[B_FIN + nuo % NSLOT], (nuo / NSLOT) & 1) &&
                               mbar_test(&bar[B_S_READY], nuo & 1) &&
                               mbar_test(&bar[B_Q_FULL + (nuo & 1)], (nuo >> 1) & 1) &&
                               (nuo < 2 || mbar_test(&bar[B_O_FREE + (nuo & 1)], ((nuo >> 1) - 1) & 1))) {
                        const int c = nuo, s = c & 1;
                        const uint32_t slot = sbase + OFF_SLOT + (c % NSLOT) * SLOT;
                        const uint32_t qst = sbase + OFF_Q + s * Q_STAGE;
                        tc_fence_after();
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            const uint32_t koff = (k >> 2) * 2 * TILE + (k & 3) * 32;
                            mma_bf16(tmem + COL_U + s * 64, smem_desc_sw128(sbase + OFF_S + koff, 16, 1024),
                                     smem_desc_sw128(slot + SL_W + k * 2048, 2 * TILE, 1024), ID_U, true);
                        }
                        mma_commit(&bar[B_U_FULL]);
                        // S-part of O with the unscaled Q; the chain applies gamma_r afterwards
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            const uint32_t koff = (k >> 2) * 2 * TILE + (k & 3) * 32;
                            const uint32_t qoff = (k >> 2) * TILE + (k & 3) * 32;
                            mma_bf16(tmem + COL_O + s * 64, smem_desc_sw128(sbase + OFF_S + koff, 16, 1024),
                                     smem_desc_sw128(qst + qoff, 16, 1024), ID_O, k > 0);
                        }
                        mma_commit(&bar[B_X_FULL]);
                        mma_commit(&bar[B_Q_EMPTY + s]);
                        GDN_TRACE_CL(c, 1, true);
                        ++nuo;
                        issued = true;
                    } else if (nwu < nchunks &&
                               mbar_test(&bar[B_BW_READY + nwu % NSLOT], (nwu / NSLOT) & 1) &&
                               mbar_test(&bar[B_V_FULL], nwu & 1) &&
                               (nwu < 2 || mbar_test(&bar[B_FIN + (nwu - 2) % NSLOT], ((nwu - 2) / NSLOT) & 1)) &&
                               (nwu < 2 || mbar_test(&bar[B_UB + (nwu & 1)], ((nwu >> 1) - 1) & 1))) {
                        const int c = nwu, s = c & 1;
                        const uint32_t slot = sbase + OFF_SLOT + (c % NSLOT) * SLOT;
                        tc_fence_after();
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            mma_bf16(tmem + COL_W + s * 64, smem_desc_sw128(slot + SL_K + k * 2048, TILE, 1024),
                                     smem_desc_sw128(slot + SL_BWT + k * 2048, 16, 1024), ID_WT, k > 0);
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            mma_bf16(tmem + COL_U + s * 64, smem_desc_sw128(sbase + OFF_V + k * 2048, TILE, 1024),
                                     smem_desc_sw128(slot + SL_X + k * 32, 16, 1024), ID_UT, k > 0);
                        mma_commit(&bar[B_W_FULL]);
                        mma_commit(&bar[B_V_EMPTY]);
                        GDN_TRACE_CL(c, 0, true);
                        ++nwu;
                        issued = true;
                    } else if (nyo < nys && mbar_test(&bar[B_O_READY + (nyo & 1)], (nyo >> 1) & 1)) {
                        const int c = nyo, s = c & 1;
                        const uint32_t slot = sbase + OFF_SLOT + (c % NSLOT) * SLOT;
                        tc_fence_after();
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            mma_bf16(tmem + COL_O + s * 64, smem_desc_sw128(sbase + OFF_U + k * 32, 16, 1024),
                                     smem_desc_sw128(slot + SL_P + k * 32, 16, 1024), ID_O, true);
                        mma_commit(&bar[B_O_FULL + s]);
                        GDN_TRACE_CL(c, 3, true);
                        ++nyo;
                        issued = true;
                    }
                    if (issued) {
                        idle_since = clock64();
                    } else {
                        __nanosleep(32);
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
            // ---------------------------------------------------- chain warpgroup
            const int q4 = warp & 3;
            const int j = q4 * 32 + lane;                 // TMEM lane = value column j
            const uint32_t t_row = tmem + ((uint32_t)(q4 * 32) << 16);
            const bool leader = (j == 0);
            (void)leader;                                 // trace builds only
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
                const int s = c & 1, sl = c % NSLOT;
                const float *gam = reinterpret_cast<const float *>(sm + OFF_SLOT + sl * SLOT + SL_VEC);
                GDN_TRACE_CL(c, 5, leader);
                if (c > 0) ok = ctl.wait(B_S_FULL, (c - 1) & 1);
                ok = ok && ctl.wait(B_RECV + sl, (c / NSLOT) & 1);
                ok = named_and(2, 128, ok);
                if (!ok) break;
                tc_fence_after();
                GDN_TRACE_CL(c, 6, leader);
                // S^T -> bf16 operand first (the U MMAs wait for it) ...
#pragma unroll 1
                for (int c0 = 0; c0 < kHeadDim; c0 += 64) {
                    float v[64];
                    tmem_ld32(t_row + COL_S + c0, v);
                    tmem_ld32(t_row + COL_S + c0 + 32, v + 32);
                    tmem_wait_ld();
                    store_row_bf16(sm + OFF_S + (c0 >> 6) * 2 * TILE, j, v);
                }
                fence_proxy_async_smem();
                mbar_arrive(&bar[B_S_READY]);
                GDN_TRACE_CL(c, 7, leader);
                // ... then S^T <- gamma_{C-1} S^T, needed only by the state MMAs of c
                const float glast = gam[C - 1];
#pragma unroll 1
                for (int c0 = 0; c0 < kHeadDim; c0 += 64) {
                    float v[64];
                    tmem_ld32(t_row + COL_S + c0, v);
                    tmem_ld32(t_row + COL_S + c0 + 32, v + 32);
                    tmem_wait_ld();
#pragma unroll
                    for (int x = 0; x < 64; ++x) v[x] *= glast;
                    tmem_st32(t_row + COL_S + c0, v);
                    tmem_st32(t_row + COL_S + c0 + 32, v + 32);
                }
                tmem_wait_st();
                // U^T -> bf16 operand, once the O MMAs of chunk c-1 have read the previous one
                ok = ctl.wait(B_U_FULL, c & 1) &&
                     (c < 1 || ctl.wait(B_O_FULL + ((c - 1) & 1), ((c - 1) >> 1) & 1));
                ok = named_and(2, 128, ok);
                if (!ok) break;
                tc_fence_after();
                GDN_TRACE_CL(c, 8, leader);
                {
                    float u[64];
                    tmem_ld32(t_row + COL_U + s * 64, u);
                    tmem_ld32(t_row + COL_U + s * 64 + 32, u + 32);
                    tmem_wait_ld();
                    store_row_bf16(sm + OFF_U, j, u);
                }
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(&bar[B_UB + s]);
                GDN_TRACE_CL(c, 9, leader);
                // S-part of O^T: column r times gamma_r (Q~ = diag(gamma) Q applied here)
                ok = named_and(2, 128, ctl.wait(B_X_FULL, c & 1));
                if (!ok) break;
                tc_fence_after();
                {
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
                tc_fence_before();
                mbar_arrive(&bar[B_O_READY + s]);
                GDN_TRACE_CL(c, 10, leader);
            }
            if (ok && nchunks > 0) ok = named_and(2, 128, ctl.wait(B_S_FULL, (nchunks - 1) & 1));
            {   // an empty sequence passes S0 (in TMEM since the start) through
                if (ok && p.S_final) {
                    tc_fence_after();
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
        } else {
            // ---------------------------------------------------- slot warpgroup
            const int pt = tid - 192;
            const int q4 = warp & 3;
            const int lrow = q4 * 32 + lane;              // TMEM lane
            const uint32_t t_row = tmem + ((uint32_t)(q4 * 32) << 16);
            const bool leader = (pt == 0);
            bool ok = true;
            // Bu and Bw^T of chunk cn out of its packed tile
            auto unpack = [&](int cn) -> bool {
                const int sl = cn % NSLOT;
                unsigned char *slot = sm + OFF_SLOT + sl * SLOT;
                GDN_TRACE_CL(cn, 30, leader);
                if (!named_and(3, 128, ctl.wait(B_RECV + sl, (cn / NSLOT) & 1))) return false;
                GDN_TRACE_CL(cn, 31, leader);
                unpack_bu_bwt(slot + SL_X, slot + SL_BWT,
                              reinterpret_cast<const float *>(slot + SL_VEC) + 128, pt);
                fence_proxy_async_smem();
                mbar_arrive(&bar[B_BW_READY + sl]);
                GDN_TRACE_CL(cn, 14, leader);
                return true;
            };
            // K tiles of chunk cn into its slot (the helper's bytes complete the slot)
            int issued_k = 0;
            auto load_k = [&](int cn) {
                const int sl = cn % NSLOT;
                unsigned char *kd = sm + OFF_SLOT + sl * SLOT + SL_K;
                mbar_arrive_expect_tx(&bar[B_RECV + sl], K_BYTES);
                tma_load_4d(kd, &tm_k, &bar[B_RECV + sl], 0, hq, sq.tb + cn * C, sq.bt);
                tma_load_4d(kd + TILE, &tm_k, &bar[B_RECV + sl], 64, hq, sq.tb + cn * C, sq.bt);
                issued_k = cn + 1;
            };
            // Chunk cp is done once its O MMAs complete: every MMA reading its slot
            // has, so the slot goes to chunk cp + 3 (K here, the rest from the
            // helper), and O^T (lane j) is stored from registers, unscaled.
            auto finish_chunk = [&](int cp) -> bool {
                const int sl = cp % NSLOT;
                if (!named_and(3, 128, ctl.wait(B_O_FULL + (cp & 1), (cp >> 1) & 1))) return false;
                tc_fence_after();
                GDN_TRACE_CL(cp, 25, leader);
                if (leader && cp + NSLOT < nchunks) {
                    load_k(cp + NSLOT);
                    remote_arrive(map_to_rank(smem_u32(&bar[B_SLOT_FREE + sl]), 1));
                }
                const uint32_t col_o = COL_O + (cp & 1) * 64;
                const int rows = min(C, sq.L - cp * C);
                const size_t row_stride = (size_t)p.Hv * kHeadDim;
                __nv_bfloat16 *dst = p.o + ((size_t)sq.bt * p.T + sq.tb + (size_t)cp * C) * row_stride +
                                     (size_t)h * kHeadDim + lrow;
                float ov[64];
                tmem_ld32(t_row + col_o, ov);
                tmem_ld32(t_row + col_o + 32, ov + 32);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(&bar[B_O_FREE + (cp & 1)]);
#pragma unroll
                for (int r = 0; r < C; ++r)
                    if (r < rows) dst[(size_t)r * row_stride] = __float2bfloat16_rn(ov[r]);
                GDN_TRACE_CL(cp, 12, leader);
                return true;
            };
            if (leader)
                for (int cn = 0; cn < NSLOT && cn < nchunks; ++cn) load_k(cn);
            if (nchunks > 0) ok = unpack(0);
            for (int c = 0; c < nchunks && ok; ++c) {
                const int sl = c % NSLOT;
                unsigned char *slot = sm + OFF_SLOT + sl * SLOT;
                // W^T (TMEM, lane d) -> W [d][r] bf16 over Bu / Bw^T; K -> K~ in place
                ok = named_and(3, 128, ctl.wait(B_W_FULL, c & 1));
                if (!ok) break;
                tc_fence_after();
                GDN_TRACE_CL(c, 11, leader);
                {
                    float w0[32], w1[32];
                    tmem_ld32(t_row + COL_W + (c & 1) * 64, w0);
                    tmem_ld32(t_row + COL_W + (c & 1) * 64 + 32, w1);
                    tmem_wait_ld();
                    GDN_TRACE_CL(c, 4, leader);
                    store_half_row_bf16(slot + SL_W, lrow, 0, w0);
                    store_half_row_bf16(slot + SL_W, lrow, 1, w1);
                }
                GDN_TRACE_CL(c, 15, leader);
                {
                    const int i = pt >> 1, half = pt & 1;
                    const float gi = reinterpret_cast<const float *>(slot + SL_VEC)[64 + i];
                    scale_row_bf16(slot + SL_K + half * TILE, slot + SL_K + half * TILE, i, gi);
                }
                GDN_TRACE_CL(c, 24, leader);
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(&bar[B_FIN + sl]);
                GDN_TRACE_CL(c, 13, leader);
                if (c + 1 < nchunks) ok = unpack(c + 1);
                if (ok && c >= 1) ok = finish_chunk(c - 1);
            }
            if (ok && nchunks > 0) ok = finish_chunk(nchunks - 1);
            if (leader && *abort_flag) {
                // let the K loads still in flight land before the CTA's memory goes away
                for (int sl = 0; sl < NSLOT && sl < issued_k; ++sl) {
                    const int c_last = sl + NSLOT * ((issued_k - 1 - sl) / NSLOT);
                    mbar_wait(&bar[B_RECV + sl], (c_last / NSLOT) & 1, 1ll << 28);
                }
            }
        }
    } else {
        // ================================================================ helper CTA
        if (warp == 0) {
            // ---------------------------------------------------- TMA: K, Q ring
            if (lane == 0) {
                bool ok = true;
                int issued = 0;
                for (int c = 0; c < nchunks && ok; ++c) {
                    const int st = c % NSTAGE, n = c / NSTAGE, t0 = sq.tb + c * C;
                    if (n >= 1) ok = ctl.wait(B_KQ_EMPTY + st, (n - 1) & 1);
                    if (!ok) break;
                    unsigned char *dst = sm + H_OFF_KQ + st * KQ_STAGE;
                    mbar_arrive_expect_tx(&bar[B_KQ_FULL + st], KQ_STAGE);
                    tma_load_4d(dst + 0 * TILE, &tm_k, &bar[B_KQ_FULL + st], 0, hq, t0, sq.bt);
                    tma_load_4d(dst + 1 * TILE, &tm_q, &bar[B_KQ_FULL + st], 0, hq, t0, sq.bt);
                    tma_load_4d(dst + 2 * TILE, &tm_k, &bar[B_KQ_FULL + st], 64, hq, t0, sq.bt);
                    tma_load_4d(dst + 3 * TILE, &tm_q, &bar[B_KQ_FULL + st], 64, hq, t0, sq.bt);
                    issued = c + 1;
                    GDN_TRACE_CL(c, 22, true);
                }
                if (*abort_flag) {
                    // let the last load into each stage land before the CTA's memory goes away
                    for (int st = 0; st < NSTAGE && st < issued; ++st) {
                        const int c_last = st + NSTAGE * ((issued - 1 - st) / NSTAGE);
                        mbar_wait(&bar[B_KQ_FULL + st], (c_last / NSTAGE) & 1, 1ll << 28);
                    }
                }
            }
        } else if (warp == 1) {
            // ---------------------------------------------------- grams, in chunk order
            if (lane == 0) {
                bool ok = true;
                for (int c = 0; c < nchunks && ok; ++c) {
                    const int st = c % NSTAGE, wg = c & 1;
                    ok = ctl.wait(B_KQ_FULL + st, (c / NSTAGE) & 1) &&
                         (c < 2 || ctl.wait(B_G_FREE + wg, ((c >> 1) - 1) & 1));
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t kq = sbase + H_OFF_KQ + st * KQ_STAGE;
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint32_t koff = (k >> 2) * 2 * TILE + (k & 3) * 32;
                        mma_bf16(tmem + wg * 64, smem_desc_sw128(kq + koff, 16, 1024),
                                 smem_desc_sw128(kq + koff, 16, 1024), ID_G, k > 0);
                    }
                    mma_commit(&bar[B_G_FULL + wg]);
                    mma_commit(&bar[B_KQ_EMPTY + st]);   // the stage's only reader
                    GDN_TRACE_CL(c, 23, true);
                }
                mma_commit(&bar[B_H_DRAIN]);
                mbar_wait(&bar[B_H_DRAIN], 0, 1ll << 30);
            }
        } else {
            // ---------------------------------------------------- prep warpgroups
            // wg 0 (warps 2-5) takes the even chunks, wg 1 (warps 6-9) the odd ones.
            const int wg = (warp - 2) >> 2;
            const int pt = tid - 64 - 128 * wg;
            const int q4 = warp & 3;
            const int row = q4 * 32 + lane;
            const int nbar = 1 + wg;
            const uint32_t t_row = tmem + ((uint32_t)(q4 * 32) << 16) + wg * 64;
            unsigned char *wgm = sm + H_OFF_WG + wg * WG_BYTES;
            float *sA = reinterpret_cast<float *>(wgm + WG_A);
            float *sY = reinterpret_cast<float *>(wgm + WG_Y);
            float *gv = reinterpret_cast<float *>(wgm + WG_GATE);
            float *vec = reinterpret_cast<float *>(wgm + WG_P + TILE);
            const int lead_warp = 2 + 4 * wg;
            bool ok = true;
            float nx_a0 = 1.f, nx_a1 = 1.f, nx_b0 = 0.f, nx_b1 = 0.f;
            if (warp == lead_warp && wg < nchunks)
                load_gates(p, sq, h, wg, lane, nx_a0, nx_a1, nx_b0, nx_b1);
            for (int c = wg, n = 0; c < nchunks && ok; c += 2, ++n) {
                GDN_TRACE_CL(c, 16, pt == 0);
                if (warp == lead_warp) {
                    const float a0 = nx_a0, a1 = nx_a1, be0 = nx_b0, be1 = nx_b1;
                    if (c + 2 < nchunks) load_gates(p, sq, h, c + 2, lane, nx_a0, nx_a1, nx_b0, nx_b1);
                    compute_gates(gv, a0, a1, be0, be1, lane);
                }
                if (pt == 0) bulk_wait_group_read0();   // the previous chunk's copies read the staging
                named_sync(nbar, 128);
                // gamma_r, g_i and beta_i gamma_i travel with the operands
                vec[pt] = pt < 64 ? gv[GV_GAM + pt] : gv[GV_G + pt - 64];
                if (pt < 64) vec[128 + pt] = gv[GV_BG + pt];
                ok = named_and(nbar, 128, ctl.wait(B_G_FULL + wg, n & 1));
                if (!ok) break;
                tc_fence_after();
                GDN_TRACE_CL(c, 17, pt == 0);
                {
                    float g0[32], g1[32];
                    tmem_ld32(t_row, g0);
                    tmem_ld32(t_row + 32, g1);
                    tmem_wait_ld();
                    tc_fence_before();
                    mbar_arrive(&bar[B_G_FREE + wg]);
                    ap_row(gv, row, g0, g1, sA, wgm + WG_P);
                }
                named_sync(nbar, 128);
                GDN_TRACE_CL(c, 18, pt == 0);
                unit_lower_inverse(sA, sY, pt, nbar);
                write_packed_bu_bwt(gv, sA, pt, wgm + WG_X);
                fence_proxy_async_smem();
                named_sync(nbar, 128);
                GDN_TRACE_CL(c, 19, pt == 0);
                if (pt == 0) {
                    // the main CTA has released the slot (from chunk c - 3)
                    const int sl = c % NSLOT;
                    ok = (c < NSLOT || ctl.wait(B_SLOT_FREE + sl, (c / NSLOT - 1) & 1));
                    GDN_TRACE_CL(c, 20, true);
                    if (ok) {
                        const uint32_t r_slot = map_to_rank(sbase + OFF_SLOT + (uint32_t)sl * SLOT, 0);
                        const uint32_t r_recv = map_to_rank(smem_u32(&bar[B_RECV + sl]), 0);
                        remote_arrive_expect_tx(r_recv, SEND_X + SEND_PV);
                        bulk_copy_to_peer(r_slot + SL_X, smem_u32(wgm + WG_X), SEND_X, r_recv);
                        bulk_copy_to_peer(r_slot + SL_P, smem_u32(wgm + WG_P), SEND_PV, r_recv);
                        bulk_commit_group();
                        GDN_TRACE_CL(c, 21, true);
                    }
                }
                ok = named_and(nbar, 128, ok);
            }
            if (pt == 0) bulk_wait_group0();
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();          // no CTA leaves while its peer may still touch its memory
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, tmem_cols);
    }
}

#ifdef GDN_TRACE
}  // namespace
// Copies the trace of the last traced launch (kTraceChunks x kTraceSlots ns stamps).
extern "C" int gdn_trace_read_cluster(unsigned long long *host, int n)
{
    if (n < kTraceChunks * kTraceSlots) return -1;
    return (int)cudaMemcpyFromSymbol(host, g_trace, sizeof(g_trace));
}
namespace {
#endif

cudaLaunchConfig_t cluster_config(int B, int Hv, cudaStream_t stream, cudaLaunchAttribute *attr)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(Hv * CLUSTER), (unsigned)B);
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = stream;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CLUSTER;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
}

}  // namespace

// True when all B * Hv clusters are resident at once (one wave): the case the
// cluster kernel is for.  The count of co-resident clusters is queried once per
// device (it depends on how the SMs split into GPCs).
bool chunk_tc_cluster_fits(int B, int Hv)
{
    constexpr int kMaxDevices = 64;
    static int resident[kMaxDevices];   // 0 = not queried yet, -1 = query failed
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return false;
    }
    if (resident[dev] == 0) {
        int n = 0;
        cudaLaunchAttribute attr[1];
        cudaLaunchConfig_t cfg = cluster_config(1, 1, nullptr, attr);
        if (cudaFuncSetAttribute(chunk_tc_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)SMEM_BYTES) != cudaSuccess ||
            cudaOccupancyMaxActiveClusters(&n, chunk_tc_cluster_kernel, &cfg) != cudaSuccess || n <= 0) {
            cudaGetLastError();   // a failed query is not an error of the next launch
            n = -1;
        }
        resident[dev] = n;
    }
    return (long long)B * Hv <= resident[dev];
}

cudaError_t launch_chunk_tc_cluster(const ChunkArgs &a, cudaStream_t stream)
{
    CUtensorMap tk, tq, tv;
    const int rows_b = a.cu_seqlens ? 1 : a.B;   // batch rows of the token arrays
    if (!make_map(&tk, a.k, rows_b, a.T, a.Hqk) || !make_map(&tq, a.q, rows_b, a.T, a.Hqk) ||
        !make_map(&tv, a.v, rows_b, a.T, a.Hv))
        return cudaErrorInvalidValue;
    cudaError_t err = cudaFuncSetAttribute(chunk_tc_cluster_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)SMEM_BYTES);
    if (err != cudaSuccess) return err;
    TcParams p{a.alpha, a.beta, a.S0, a.S_final, a.T, a.Hqk, a.Hv,
               static_cast<__nv_bfloat16 *>(a.o), a.cu_seqlens};
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = cluster_config(a.B, a.Hv, stream, attr);
    err = cudaLaunchKernelEx(&cfg, chunk_tc_cluster_kernel, tk, tq, tv, p);
    if (err != cudaSuccess) return err;
    return cudaGetLastError();
}

}  // namespace gdn
