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
//   3. fix_tc_kernel adds R S_start(k) to the outputs of segment k >= 1 on the
//      tensor core (tcgen05, fp32 accumulation in TMEM, one rounding to bf16).
// With two segments, S_start(1) = D_0: the chunk kernel writes its bf16 transpose
// itself, so step 2 shrinks to the final state M_1 D_0 + D_1 (split2_state_kernel,
// only when the caller asks for it) and the fix-up no longer waits for it.
// The serial chain of chunk steps is one segment long instead of the sequence.
#include "tc_common.cuh"

namespace gdn {
namespace {

constexpr int kChainThreads = 256;
constexpr int kChainCols = 32;            // state columns per CTA of seg_chain_kernel
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

// Two segments: the final state M_1 D_0 + D_1, kStateCols columns of one (head,
// sequence) per CTA.
constexpr int kStateCols = 16;            // 128 threads: one 4 x 4 tile each
__global__ void __launch_bounds__(128)
split2_state_kernel(const float *__restrict__ segD, const float *__restrict__ segM, float *S_final, int Hv)
{
    extern __shared__ __align__(16) float state_smem[];
    constexpr int per_head = kHeadDim / kStateCols;
    const int jb = blockIdx.x % per_head, bh = blockIdx.x / per_head;
    chain_columns<128, kStateCols>(segD, segM, nullptr, S_final, 2, Hv, bh % Hv, bh / Hv, jb * kStateCols,
                                   false, state_smem);
}

// o[t] += R[t - seg_len] S_start(k) for 128 rows of segment k >= 1 of one (sequence,
// V head), on the tensor core.  The R rows (A: rows t, K = d) and S_start(k)^T (B:
// rows j, K = d; both K-major) come in by TMA, 32 KB each as four 64 x 64 bf16 boxes
// in the 128-byte swizzle; eight tcgen05 MMAs (M = N = 128, K = 16 each) accumulate
// in TMEM; thread r reads row r back, adds the chunk kernel's o^0 and writes one bf16
// rounding.  R rows past the segment or the sequence are loaded (zero past the end of
// R) but not stored.  CTA x: tile x % tps of segment 1 + (x / tps) % (nseg - 1) of
// (sequence, head) x / (tps (nseg - 1)), tps = ceil(seg_len / 128).
constexpr int kFixTcRows = 128;
constexpr uint32_t kFixTcTile = 64 * 64 * 2;                // one 64 x 64 bf16 box
constexpr uint32_t kFixTcSmem = 8 * kFixTcTile + 64 + 1024; // A, B, barriers + flag, alignment

__global__ void __launch_bounds__(128, 1)
fix_tc_kernel(const __grid_constant__ CUtensorMap tm_r, const __grid_constant__ CUtensorMap tm_s,
              __nv_bfloat16 *__restrict__ o, int T, int seg_len, int nseg, int Hv)
{
    extern __shared__ __align__(1024) unsigned char fix_raw[];
    const int tps = (seg_len + kFixTcRows - 1) / kFixTcRows;
    const int x = blockIdx.x;
    const int tile = x % tps, km1 = (x / tps) % (nseg - 1), bh = x / (tps * (nseg - 1));
    const int h = bh % Hv, b = bh / Hv;
    const int TR = T - seg_len;                                      // rows of R
    const int r0 = km1 * seg_len + tile * kFixTcRows;                // first R row of the tile
    const int r_end = min(min(r0 + kFixTcRows, (km1 + 1) * seg_len), TR);
    if (r0 >= r_end) return;                                         // a tile past a short last segment
    unsigned char *sm = fix_raw + ((1024u - (smem_u32(fix_raw) & 1023u)) & 1023u);
    unsigned char *sA = sm, *sB = sm + 4 * kFixTcTile;
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + 8 * kFixTcTile);   // 0: loads, 1: MMAs
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + 8 * kFixTcTile + 16);
    volatile int *s_ok = reinterpret_cast<volatile int *>(sm + 8 * kFixTcTile + 32);
    const int tid = threadIdx.x, warp = tid >> 5;
    if (tid == 0) {
        prefetch_tensormap(&tm_r);
        prefetch_tensormap(&tm_s);
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (tid == 0) {
        mbar_arrive_expect_tx(&bar[0], 8 * kFixTcTile);
        const int srow = ((b * (nseg - 1) + km1) * Hv + h) * kHeadDim;   // S_start(k)^T row j = 0
#pragma unroll
        for (int q = 0; q < 4; ++q) {   // box q: d-half q >> 1, 64-row half q & 1
            tma_load_4d(sA + q * kFixTcTile, &tm_r, &bar[0], 64 * (q >> 1), h, r0 + 64 * (q & 1), b);
            tma_load_4d(sB + q * kFixTcTile, &tm_s, &bar[0], 64 * (q >> 1), 0, srow + 64 * (q & 1), 0);
        }
        const bool loaded = mbar_wait(&bar[0], 0, 1ll << 30);
        if (loaded) {
            tc_fence_after();
            constexpr uint32_t idesc = idesc_bf16(128, 128, false, false);
#pragma unroll
            for (int k = 0; k < 8; ++k) {   // K-step k: d 16k .. 16k+15
                const uint32_t off = (k >> 2) * 2 * kFixTcTile + (k & 3) * 32;
                mma_bf16(tmem, smem_desc_sw128(smem_u32(sA) + off, 16, 1024),
                         smem_desc_sw128(smem_u32(sB) + off, 16, 1024), idesc, k > 0);
            }
        } else {
            atomicOr(&g_tc_error, 1u);
        }
        *s_ok = loaded ? 1 : 0;
        mma_commit(&bar[1]);   // with no MMA issued it arrives at once
    }
    // thread r: row r of the tile (TMEM lane r) -> o[b][seg_len + r0 + r][h][:]
    const int r = tid;
    const bool live = r0 + r < r_end;
    const size_t row_stride = (size_t)Hv * kHeadDim;
    uint4 *orow = reinterpret_cast<uint4 *>(o + ((size_t)b * T + seg_len + r0 + r) * row_stride +
                                            (size_t)h * kHeadDim);
    uint4 old[16];
    if (live) {
#pragma unroll
        for (int c = 0; c < 16; ++c) old[c] = orow[c];
    }
    __syncthreads();   // *s_ok written
    const bool done = mbar_wait(&bar[1], 0, 1ll << 30);
    if (!done && tid == 0) atomicOr(&g_tc_error, 1u);
    const bool store = live && done && *s_ok;
    tc_fence_after();
    const uint32_t t_row = tmem + ((uint32_t)(32 * warp) << 16);
#pragma unroll
    for (int c = 0; c < 4; ++c) {   // columns j 32c .. 32c+31
        float acc[32];
        tmem_ld32(t_row + 32 * c, acc);
        tmem_wait_ld();
        if (store) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const __nv_bfloat162 *ov = reinterpret_cast<const __nv_bfloat162 *>(&old[4 * c + q]);
                uint32_t pk[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = __bfloat1622float2(ov[e]);
                    pk[e] = pack_bf16x2(f.x + acc[8 * q + 2 * e], f.y + acc[8 * q + 2 * e + 1]);
                }
                orow[4 * c + q] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

// Launches fix_tc_kernel over every later segment's rows.
cudaError_t launch_fix_tc(const ChunkArgs &a, int seg_len, int nseg, const __nv_bfloat16 *R,
                          const __nv_bfloat16 *sstT, cudaStream_t stream)
{
    CUtensorMap tr, ts;
    if (!make_map(&tr, R, a.B, a.T - seg_len, a.Hv) ||
        !make_map(&ts, sstT, 1, a.B * (nseg - 1) * a.Hv * kHeadDim, 1))
        return cudaErrorInvalidValue;
    cudaError_t err = cudaFuncSetAttribute(fix_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)kFixTcSmem);
    if (err != cudaSuccess) return err;
    const int tps = (seg_len + kFixTcRows - 1) / kFixTcRows;
    fix_tc_kernel<<<(unsigned)(a.B * a.Hv * (nseg - 1) * tps), 128, kFixTcSmem, stream>>>(
        tr, ts, static_cast<__nv_bfloat16 *>(a.o), a.T, seg_len, nseg, a.Hv);
    return cudaGetLastError();
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

    if (pl.nseg == 2) {
        cudaError_t err = launch_chunk_tc_segments(a, pl.seg_len, pl.nseg, segD, segM, R, sstT, stream);
        if (err != cudaSuccess) return err;
        if (a.S_final) {   // the final state M_1 D_0 + D_1 (fp32, CUDA cores)
            const size_t smem = ((size_t)kHeadDim * kLdM + (size_t)kHeadDim * kStateCols) * sizeof(float);
            err = cudaFuncSetAttribute(split2_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
            if (err != cudaSuccess) return err;
            split2_state_kernel<<<(unsigned)(a.B * a.Hv * (kHeadDim / kStateCols)), 128, smem, stream>>>(
                segD, segM, a.S_final, a.Hv);
            err = cudaGetLastError();
            if (err != cudaSuccess) return err;
        }
        return launch_fix_tc(a, pl.seg_len, pl.nseg, R, sstT, stream);
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
    return launch_fix_tc(a, pl.seg_len, pl.nseg, R, sstT, stream);
}

// Reads and clears this file's error word (bit 0: a bounded wait of the fix-up gave up).
cudaError_t split_take_error(unsigned *out)
{
    unsigned v = 0, zero = 0;
    cudaError_t err = cudaMemcpyFromSymbol(&v, g_tc_error, sizeof(v));
    if (err == cudaSuccess && v) err = cudaMemcpyToSymbol(g_tc_error, &zero, sizeof(zero));
    *out = v;
    return err;
}

}  // namespace gdn
