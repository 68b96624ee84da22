// Device code shared by the tensor-core prefill kernels (one CTA per head, and the
// pipelined kernel's prep and chain CTAs): constants, bf16 operand writers, barrier helpers, the blocked
// triangular inverse, gate loading, and the host-side TMA descriptor builder.
// Everything is in an anonymous namespace: each kernel file gets its own copy.
#pragma once

#include <cuda.h>

#include "gdn_internal.cuh"
#include "sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

__device__ unsigned int g_tc_error = 0;   // set when a bounded wait gave up (per kernel file)

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


constexpr int C = kChunk;          // 64
constexpr uint32_t TILE = 8192;    // one 64 x 64 bf16 tile, 128B-swizzled
constexpr int LDA = 68;            // padded row stride (floats) of the fp32 A / T matrix
constexpr int LDY = 40;            // row stride of the solve scratch
// per-chunk gate vectors: b (log2 units), gamma, beta, g, beta*gamma, alpha (as used:
// 2^(clamped log2 alpha)), and d31[i] = prod_{i<j<=31} alpha_j (i < 32)
constexpr int GV_B = 0, GV_GAM = 64, GV_BETA = 128, GV_G = 192, GV_BG = 256, GV_ALPHA = 320,
              GV_D31 = 384;
constexpr uint32_t GATE_BUF = 416 * 4;

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
    __nv_bfloat16 *o;   // output, for stores without a tensor map
    const int *cu_seqlens;   // packed sequences (see ChunkArgs), or null
    // Segment mode (seg_len > 0): each of the B sequences is cut into nseg segments
    // of seg_len tokens.  CTA rows y < B*nseg run segment y % nseg of sequence
    // y / nseg from its start state (S0 for the first segment, zero otherwise),
    // writing o and its final state to seg_D; the B*(nseg-1) rows after them run
    // segments 1.. from S = I with v = 0, writing their outputs (M_t^T q_t) through
    // the second output map (or r) and their final state (the segment's
    // transition) to seg_M.
    int B, seg_len, nseg;
    float *seg_D, *seg_M;
    __nv_bfloat16 *r;   // transition-row outputs [B, T - seg_len, Hv, 128], segment mode
    __nv_bfloat16 *sst; // segment mode, or null: S_start(1)^T = bf16 of the first
                        // segment's final state, transposed, [B, Hv, 128 (j), 128 (d)]
    int l2_prefetch;    // 1: pull each K/Q/V tile into L2 a few chunks before its load
};

// Token rows of sequence b: rows tb .. tb + L of batch row bt of the token arrays.
struct SeqSpan {
    int tb, L, bt;
};
__device__ __forceinline__ SeqSpan seq_span(const TcParams &p, int b) {
    if (!p.cu_seqlens) return SeqSpan{0, p.T, b};
    const int s0 = min(max(p.cu_seqlens[b], 0), p.T);   // clamped into [0, T]
    const int s1 = min(max(p.cu_seqlens[b + 1], s0), p.T);
    return SeqSpan{s0, s1 - s0, 0};
}

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

// alpha, beta of tokens 2*lane, 2*lane+1 of chunk cn of the sequence (alpha = 1,
// beta = 0 past its end: those rows then add nothing to the state)
__device__ __forceinline__ void load_gates(const TcParams &p, const SeqSpan &sq, int h, int cn, int lane,
                                           float &a0, float &a1, float &b0, float &b1) {
    const int tn = cn * C, Ln = min(C, sq.L - tn);
    const int r = 2 * lane;
    const size_t gi = ((size_t)sq.bt * p.T + sq.tb + tn + r) * p.Hv + h;
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


// ---------------------------------------------------------------- shared prep steps
// Gate vectors of one chunk into gv (warp-wide: lane holds tokens 2*lane, 2*lane+1):
// alpha a0/a1 and beta be0/be1 of those tokens (alpha = 1, beta = 0 past the end).
__device__ __forceinline__ void compute_gates(float *gv, float a0, float a1, float be0, float be1,
                                              int lane) {
    // log2 alpha, clamped at -87 / ln 2 (alpha = 0 stays finite)
    const float la0 = fmaxf(fast_log2(a0), kLog2Floor);
    const float la1 = fmaxf(fast_log2(a1), kLog2Floor);
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

// One row of A (row < 64: beta_r Gam[r][i] k_r.k_i for i < r, fp32 into sA) or of P
// (row >= 64: Gam[r][i] q_r.k_i for i <= r, bf16 into the P tile), from the gram row
// g0 (columns 0-31) / g1 (32-63) held by this thread.  Decay factors are running
// products of alpha along the row, Gam[r][x-1] = Gam[r][x] alpha_x from x = r down;
// rows r >= 32 continue into columns x < 32 with d31[x] = Gam[31][x].
// (ap_row_values computes the row in place in g0 / g1; ap_row also stores it.)
__device__ __forceinline__ void ap_row_values(const float *gv, int row, float *g0, float *g1) {
    const int r = row & 63;
    const bool is_a = row < 64;                // A rows: strict lower; P rows: i <= r
    const bool low = r < 32;                   // warp-uniform
    float run = is_a ? gv[GV_BETA + r] : 1.f;  // row scale folded into the product
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
}
__device__ __forceinline__ void ap_row(const float *gv, int row, float *g0, float *g1, float *sA,
                                       unsigned char *ptile) {
    ap_row_values(gv, row, g0, g1);
    const int r = row & 63;
    if (row < 64) {
        float4 *dst = reinterpret_cast<float4 *>(sA + r * LDA);
#pragma unroll
        for (int x = 0; x < 8; ++x) dst[x] = make_float4(g0[4 * x], g0[4 * x + 1], g0[4 * x + 2], g0[4 * x + 3]);
#pragma unroll
        for (int x = 0; x < 8; ++x) dst[8 + x] = make_float4(g1[4 * x], g1[4 * x + 1], g1[4 * x + 2], g1[4 * x + 3]);
    } else {
        store_half_row_bf16(ptile, r, 0, g0);
        store_half_row_bf16(ptile, r, 1, g1);
    }
}

// Bw = T diag(beta gamma) (threads pt 0-63, row pt) and Bu = T diag(beta)
// (pt 64-127, row pt - 64) as bf16 operand tiles, from T in sA.
__device__ __forceinline__ void write_bw_bu(const float *gv, const float *sA, int pt,
                                            unsigned char *bw, unsigned char *bu) {
    const int r = pt & 63;
    unsigned char *dst = pt < 64 ? bw : bu;
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
}  // namespace gdn
