// Segment-parallel prefill (T-split) for sequences too few to fill the GPU.
//
// The update of "Qwen3.8-Flash-Next 技术总结 -- Qwen4 架构的探路者", section 2.1
// "Gated DeltaNet", S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,
// is affine in the state.  Over a segment of tokens it is therefore
//   S_t = M_t S_start + D_t,   o_t = S_t^T q_t = D_t^T q_t + S_start^T (M_t^T q_t),
// where D_t is the state reached from a zero start with the real v, and M_t the
// state reached from S = I with v = 0.  So each sequence is cut into segments run
// side by side:
//   1. one launch of the chunk kernel runs every segment from a zero start (the
//      first from S0), giving o^0 and D = D_end, and every later segment from
//      S = I with v = 0, giving R (rows r_t = M_t^T q_t) and M = M_end;
//   2. seg_chain_kernel walks the segments of each (sequence, head):
//      S_start(k+1) = M_k S_start(k) + D_k in fp32, keeping every S_start(k)^T
//      in bf16;
//   3. out_fix_kernel adds R S_start(k) to the outputs of segment k >= 1
//      (bf16 warp MMAs, fp32 accumulation, one rounding to bf16).
// With two segments, S_start(1) = D_0: the chunk kernel writes its bf16 transpose
// itself, and the fix-up and the final state M_1 D_0 + D_1 no longer depend on
// each other, so one launch (split2_finish_kernel) runs both side by side.
// The serial chain of chunk steps is one segment long instead of the sequence.
#include "tc_common.cuh"

namespace gdn {
namespace {

constexpr int kChainThreads = 256;
constexpr int kChainCols = 32;            // state columns per CTA of seg_chain_kernel
constexpr int kFixRows = 64;              // output rows per tile of out_fix_kernel
constexpr int kFixTiles = 2;              // tiles per CTA (the S_start tile is staged once)
constexpr int kLdR = kHeadDim + 8;        // padded bf16 row strides in shared memory
constexpr int kLdS = kHeadDim + 8;
constexpr int kLdM = kHeadDim + 1;        // padded row stride of the staged M (floats): the
                                          // threads of a warp read rows i0 + x at one d, in
                                          // distinct banks

// S_start of every later segment, in order: S_start(1) = D_0, S_start(k+1) =
// M_k S_start(k) + D_k (fp32); writes S_start(k)^T in bf16 ([j][d]) for k >= 1 if
// write_sst, and the final state.  Columns of the state evolve independently, so
// one CTA of kThreads threads takes kCols columns of one (head, sequence): M_k
// whole and its columns of S in shared memory (chain_smem, kHeadDim * (kLdM +
// kCols) floats); each thread owns a 4 x 4 tile of the product.
template <int kThreads, int kCols>
__device__ __forceinline__ void chain_columns(const float *__restrict__ segD, const float *__restrict__ segM,
                                              __nv_bfloat16 *__restrict__ sstT, float *S_final, int nseg,
                                              int Hv, int h, int b, int j_base, bool write_sst,
                                              float *chain_smem)
{
    static_assert((kHeadDim / 4) * (kCols / 4) == kThreads, "one 4 x 4 tile per thread");
    float *Ms = chain_smem;                        // M_k: [i][d], row stride kLdM
    float *Sc = chain_smem + kHeadDim * kLdM;      // S_start columns: [d][c], c < kCols
    const int tid = threadIdx.x;
    const size_t hs = (size_t)kHeadDim * kHeadDim;
    const float *D0 = segD + (((size_t)b * nseg + 0) * Hv + h) * hs;
#pragma unroll 16
    for (int e = tid; e < kHeadDim * kCols; e += kThreads) {
        const int d = e / kCols, c = e % kCols;
        Sc[e] = D0[(size_t)d * kHeadDim + j_base + c];
    }
    // thread tile: rows i0 .. i0+3 (of 128), columns c0 .. c0+3 (of kCols)
    const int i0 = 4 * (tid / (kCols / 4)), c0 = 4 * (tid % (kCols / 4));
    for (int k = 1; k < nseg; ++k) {
        const float *Mk = segM + (((size_t)b * (nseg - 1) + (k - 1)) * Hv + h) * hs;
        const float *Dk = segD + (((size_t)b * nseg + k) * Hv + h) * hs;
        __nv_bfloat16 *dst = sstT + (((size_t)b * (nseg - 1) + (k - 1)) * Hv + h) * hs;
        __syncthreads();                           // Sc complete; Ms free
#pragma unroll 16
        for (int e = tid; e < kHeadDim * kHeadDim / 4; e += kThreads) {
            const float4 v = reinterpret_cast<const float4 *>(Mk)[e];
            float *row = Ms + (e / (kHeadDim / 4)) * kLdM + 4 * (e % (kHeadDim / 4));
            row[0] = v.x; row[1] = v.y; row[2] = v.z; row[3] = v.w;
        }
        // S_start(k)^T for the output fix-up: row j = j_base + c, 128 bf16 (d)
        for (int e = tid; write_sst && e < kCols * (kHeadDim / 8); e += kThreads) {
            const int c = e / (kHeadDim / 8), d8 = 8 * (e % (kHeadDim / 8));
            __align__(16) __nv_bfloat16 v8[8];
#pragma unroll
            for (int x = 0; x < 8; ++x) v8[x] = __float2bfloat16_rn(Sc[(d8 + x) * kCols + c]);
            *reinterpret_cast<uint4 *>(dst + (size_t)(j_base + c) * kHeadDim + d8) =
                *reinterpret_cast<const uint4 *>(v8);
        }
        __syncthreads();
        float acc[4][4];
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
            for (int y = 0; y < 4; ++y) acc[x][y] = 0.f;
#pragma unroll 4
        for (int d = 0; d < kHeadDim; ++d) {
            float mi[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) mi[x] = Ms[(i0 + x) * kLdM + d];
            const float4 sv = *reinterpret_cast<const float4 *>(&Sc[d * kCols + c0]);
            const float sj[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(mi[x], sj[y], acc[x][y]);
        }
        __syncthreads();                           // every thread has read Sc
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const float4 dv = *reinterpret_cast<const float4 *>(&Dk[(size_t)(i0 + x) * kHeadDim + j_base + c0]);
            *reinterpret_cast<float4 *>(&Sc[(i0 + x) * kCols + c0]) =
                make_float4(acc[x][0] + dv.x, acc[x][1] + dv.y, acc[x][2] + dv.z, acc[x][3] + dv.w);
        }
    }
    __syncthreads();
    if (S_final) {
        float *out = S_final + ((size_t)b * Hv + h) * hs;
#pragma unroll 16
        for (int e = tid; e < kHeadDim * kCols; e += kThreads) {
            const int d = e / kCols, c = e % kCols;
            out[(size_t)d * kHeadDim + j_base + c] = Sc[e];
        }
    }
}

__global__ void __launch_bounds__(kChainThreads, 1)
seg_chain_kernel(const float *__restrict__ segD, const float *__restrict__ segM,
                 __nv_bfloat16 *__restrict__ sstT, float *S_final, int nseg, int Hv)
{
    extern __shared__ __align__(16) float chain_smem[];
    chain_columns<kChainThreads, kChainCols>(segD, segM, sstT, S_final, nseg, Hv, blockIdx.x, blockIdx.y,
                                             blockIdx.z * kChainCols, true, chain_smem);
}

__device__ __forceinline__ uint32_t ld_u32(const __nv_bfloat16 *p) {
    return *reinterpret_cast<const uint32_t *>(p);
}

// o[t] += R[t - seg_len] S_start(k) for the rows t of segment k >= 1.  One CTA of
// 128 threads per kFixTiles x kFixRows rows (row group `grp`, counting the groups
// of every later segment in order) of one (head, sequence); 4 warps of 16 rows x
// 128 columns per tile.
__device__ __forceinline__ void fix_rows(const __nv_bfloat16 *__restrict__ Rr,
                                         const __nv_bfloat16 *__restrict__ sstT,
                                         __nv_bfloat16 *__restrict__ o, int T, int seg_len, int nseg,
                                         int Hv, int grp, int h, int b, __nv_bfloat16 *fix_smem)
{
    __nv_bfloat16 *sS = fix_smem;                        // S_start^T: [j][kLdS]
    __nv_bfloat16 *sR = fix_smem + kHeadDim * kLdS;      // R tile: [kFixRows][kLdR]
    __nv_bfloat16 *sO = sR + kFixRows * kLdR;            // o tile: [kFixRows][kLdR]
    const int tid = threadIdx.x;
    const int TR = T - seg_len;                          // rows of R
    const int groups = (seg_len + kFixTiles * kFixRows - 1) / (kFixTiles * kFixRows);
    const int k = 1 + grp / groups;                      // segment
    const int seg_r0 = (k - 1) * seg_len;                // its first R row
    const int r_begin = seg_r0 + (grp % groups) * kFixTiles * kFixRows;
    const int r_end = min(min(r_begin + kFixTiles * kFixRows, seg_r0 + seg_len), TR);
    const size_t row_stride = (size_t)Hv * kHeadDim;
    const __nv_bfloat16 *St = sstT + (((size_t)b * (nseg - 1) + (k - 1)) * Hv + h) * kHeadDim * kHeadDim;
#pragma unroll 16
    for (int e = tid; e < kHeadDim * (kHeadDim / 8); e += 128) {
        const int j = e / (kHeadDim / 8), c8 = e % (kHeadDim / 8);
        *reinterpret_cast<uint4 *>(&sS[j * kLdS + 8 * c8]) =
            *reinterpret_cast<const uint4 *>(St + (size_t)j * kHeadDim + 8 * c8);
    }
    const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, tq = lane & 3;
    for (int r0 = r_begin; r0 < r_end; r0 += kFixRows) {
        __syncthreads();                                 // sS staged; previous tile stored
        // R rows and the matching o^0 rows (o row of R row rr is rr + seg_len), 16-byte
        // coalesced loads; rows past the segment are zero / not stored
#pragma unroll 8
        for (int e = tid; e < kFixRows * (kHeadDim / 8); e += 128) {
            const int r = e / (kHeadDim / 8), c8 = e % (kHeadDim / 8);
            uint4 v = make_uint4(0u, 0u, 0u, 0u), w = v;
            if (r0 + r < r_end) {
                v = *reinterpret_cast<const uint4 *>(Rr + ((size_t)b * TR + r0 + r) * row_stride +
                                                     (size_t)h * kHeadDim + 8 * c8);
                w = *reinterpret_cast<const uint4 *>(o + ((size_t)b * T + r0 + r + seg_len) * row_stride +
                                                     (size_t)h * kHeadDim + 8 * c8);
            }
            *reinterpret_cast<uint4 *>(&sR[r * kLdR + 8 * c8]) = v;
            *reinterpret_cast<uint4 *>(&sO[r * kLdR + 8 * c8]) = w;
        }
        __syncthreads();
        // the accumulators start from o^0
        float acc[16][4];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const __nv_bfloat16 *orow = &sO[(16 * warp + g + 8 * half) * kLdR];
#pragma unroll
            for (int n = 0; n < 16; ++n) {
                const float2 cur = __bfloat1622float2(
                    *reinterpret_cast<const __nv_bfloat162 *>(orow + 8 * n + 2 * tq));
                acc[n][2 * half] = cur.x;
                acc[n][2 * half + 1] = cur.y;
            }
        }
        const __nv_bfloat16 *a_lo = &sR[(16 * warp + g) * kLdR];
        const __nv_bfloat16 *a_hi = &sR[(16 * warp + g + 8) * kLdR];
#pragma unroll
        for (int ks = 0; ks < kHeadDim / 16; ++ks) {
            const int kc = 16 * ks + 2 * tq;
            const uint32_t a0 = ld_u32(a_lo + kc), a1 = ld_u32(a_hi + kc);
            const uint32_t a2 = ld_u32(a_lo + kc + 8), a3 = ld_u32(a_hi + kc + 8);
#pragma unroll
            for (int n = 0; n < 16; ++n) {
                const __nv_bfloat16 *bp = &sS[(8 * n + g) * kLdS + kc];
                const uint32_t b0 = ld_u32(bp), b1 = ld_u32(bp + 8);
                asm volatile(
                    "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
                    "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                    : "+f"(acc[n][0]), "+f"(acc[n][1]), "+f"(acc[n][2]), "+f"(acc[n][3])
                    : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
            }
        }
        // results back into the o tile (each warp its own 16 rows), then 16-byte stores
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            __nv_bfloat16 *orow = &sO[(16 * warp + g + 8 * half) * kLdR];
#pragma unroll
            for (int n = 0; n < 16; ++n)
                *reinterpret_cast<__nv_bfloat162 *>(orow + 8 * n + 2 * tq) =
                    __floats2bfloat162_rn(acc[n][2 * half], acc[n][2 * half + 1]);
        }
        __syncthreads();
#pragma unroll 8
        for (int e = tid; e < kFixRows * (kHeadDim / 8); e += 128) {
            const int r = e / (kHeadDim / 8), c8 = e % (kHeadDim / 8);
            if (r0 + r < r_end)
                *reinterpret_cast<uint4 *>(o + ((size_t)b * T + r0 + r + seg_len) * row_stride +
                                           (size_t)h * kHeadDim + 8 * c8) =
                    *reinterpret_cast<const uint4 *>(&sO[r * kLdR + 8 * c8]);
        }
    }
}

__global__ void __launch_bounds__(128)
out_fix_kernel(const __nv_bfloat16 *__restrict__ Rr, const __nv_bfloat16 *__restrict__ sstT,
               __nv_bfloat16 *__restrict__ o, int T, int seg_len, int nseg, int Hv)
{
    extern __shared__ __align__(16) __nv_bfloat16 fix_smem[];
    fix_rows(Rr, sstT, o, T, seg_len, nseg, Hv, blockIdx.x, blockIdx.y, blockIdx.z, fix_smem);
}

// Two segments: CTAs [0, n_state) compute the final state M_1 D_0 + D_1 (kStateCols
// columns of one (head, sequence) each), the rest the output fix-up of segment 1,
// whose S_start(1)^T the chunk kernel has written.
constexpr int kStateCols = 16;            // 128 threads: one 4 x 4 tile each
__global__ void __launch_bounds__(128)
split2_finish_kernel(const float *__restrict__ segD, const float *__restrict__ segM,
                     const __nv_bfloat16 *__restrict__ Rr, const __nv_bfloat16 *__restrict__ sstT,
                     __nv_bfloat16 *__restrict__ o, float *S_final, int T, int seg_len, int Hv, int B)
{
    extern __shared__ __align__(16) unsigned char finish_smem[];
    constexpr int per_head = kHeadDim / kStateCols;
    const int n_state = S_final ? B * Hv * per_head : 0;
    const int x = blockIdx.x;
    if (x < n_state) {
        const int jb = x % per_head, bh = x / per_head;
        chain_columns<128, kStateCols>(segD, segM, nullptr, S_final, 2, Hv, bh % Hv, bh / Hv,
                                       jb * kStateCols, false, reinterpret_cast<float *>(finish_smem));
        return;
    }
    const int groups = (seg_len + kFixTiles * kFixRows - 1) / (kFixTiles * kFixRows);
    const int y = x - n_state;                           // (b, h, group)
    fix_rows(Rr, sstT, o, T, seg_len, 2, Hv, y % groups, (y / groups) % Hv, y / (groups * Hv),
             reinterpret_cast<__nv_bfloat16 *>(finish_smem));
}

constexpr size_t align_up(size_t x) { return (x + 1023) & ~(size_t)1023; }

struct SplitPlan {
    int seg_len, nseg;
    size_t off_D, off_M, off_R, off_S, bytes;
};

SplitPlan plan_split(int B, int T, int Hv, int segments)
{
    SplitPlan pl{};
    const int nchunks = (T + kChunk - 1) / kChunk;
    const int seg_chunks = (nchunks + segments - 1) / segments;
    pl.seg_len = seg_chunks * kChunk;
    pl.nseg = (T + pl.seg_len - 1) / pl.seg_len;
    const size_t hs = (size_t)kHeadDim * kHeadDim;
    const size_t nlater = pl.nseg > 1 ? (size_t)pl.nseg - 1 : 0;
    pl.off_D = 0;
    pl.off_M = align_up(pl.off_D + (size_t)B * pl.nseg * Hv * hs * sizeof(float));
    pl.off_R = align_up(pl.off_M + (size_t)B * nlater * Hv * hs * sizeof(float));
    const size_t r_rows = pl.nseg > 1 ? (size_t)(T - pl.seg_len) : 0;
    pl.off_S = align_up(pl.off_R + (size_t)B * r_rows * Hv * kHeadDim * sizeof(__nv_bfloat16));
    pl.bytes = align_up(pl.off_S + (size_t)B * nlater * Hv * hs * sizeof(__nv_bfloat16));
    return pl;
}

}  // namespace

size_t chunk_tc_split_workspace(int B, int T, int Hv, int segments)
{
    if (B <= 0 || T <= 0 || segments <= 1) return 0;
    const SplitPlan pl = plan_split(B, T, Hv, segments);
    return pl.nseg > 1 ? pl.bytes : 0;
}

cudaError_t launch_chunk_tc_split(const ChunkArgs &a, int segments, void *workspace, cudaStream_t stream)
{
    const SplitPlan pl = plan_split(a.B, a.T, a.Hv, segments);
    if (pl.nseg <= 1) return launch_chunk_tc(a, stream);
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    float *segD = reinterpret_cast<float *>(ws + pl.off_D);
    float *segM = reinterpret_cast<float *>(ws + pl.off_M);
    __nv_bfloat16 *R = reinterpret_cast<__nv_bfloat16 *>(ws + pl.off_R);
    __nv_bfloat16 *sstT = reinterpret_cast<__nv_bfloat16 *>(ws + pl.off_S);

    const size_t fix_smem = (size_t)(2 * kFixRows * kLdR + kHeadDim * kLdS) * sizeof(__nv_bfloat16);
    const int groups = (pl.seg_len + kFixTiles * kFixRows - 1) / (kFixTiles * kFixRows);
    if (pl.nseg == 2) {
        cudaError_t err = launch_chunk_tc_segments(a, pl.seg_len, pl.nseg, segD, segM, R, sstT, stream);
        if (err != cudaSuccess) return err;
        const size_t state_smem = ((size_t)kHeadDim * kLdM + (size_t)kHeadDim * kStateCols) * sizeof(float);
        const size_t smem = state_smem > fix_smem ? state_smem : fix_smem;
        err = cudaFuncSetAttribute(split2_finish_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
        const int n_state = a.S_final ? a.B * a.Hv * (kHeadDim / kStateCols) : 0;
        split2_finish_kernel<<<(unsigned)(n_state + a.B * a.Hv * groups), 128, smem, stream>>>(
            segD, segM, R, sstT, static_cast<__nv_bfloat16 *>(a.o), a.S_final, a.T, pl.seg_len, a.Hv, a.B);
        return cudaGetLastError();
    }
    cudaError_t err = launch_chunk_tc_segments(a, pl.seg_len, pl.nseg, segD, segM, R, nullptr, stream);
    if (err != cudaSuccess) return err;
    const size_t chain_smem = ((size_t)kHeadDim * kLdM + (size_t)kHeadDim * kChainCols) * sizeof(float);
    err = cudaFuncSetAttribute(seg_chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)chain_smem);
    if (err != cudaSuccess) return err;
    seg_chain_kernel<<<dim3((unsigned)a.Hv, (unsigned)a.B, kHeadDim / kChainCols), kChainThreads,
                       chain_smem, stream>>>(segD, segM, sstT, a.S_final, pl.nseg, a.Hv);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    // each CTA covers up to kFixTiles x kFixRows rows of one segment
    err = cudaFuncSetAttribute(out_fix_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fix_smem);
    if (err != cudaSuccess) return err;
    out_fix_kernel<<<dim3((unsigned)((pl.nseg - 1) * groups), (unsigned)a.Hv, (unsigned)a.B),
                     128, fix_smem, stream>>>(R, sstT, static_cast<__nv_bfloat16 *>(a.o), a.T, pl.seg_len,
                                       pl.nseg, a.Hv);
    return cudaGetLastError();
}

}  // namespace gdn
