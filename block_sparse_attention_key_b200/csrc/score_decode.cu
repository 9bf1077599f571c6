// Indexer block scores for decode-shaped calls (step 2 of the QSA layer).
//
// blog.cecily.jp/6295 (Raschka's explainer paragraph): a learned indexer rates
// every block from its averaged key; keieiax.jp glossary "Qwen Sparse Attention",
// section on 4-token micro-blocks: the indexer estimates each block's importance.
// The score of block b for query i is
//     sum_h w[i][h] * ReLU( q_idx[i][h] . pooled[s][b] )        (4 heads x 64 dims)
// over the complete causal blocks b < floor((t+1)/bs) (bs = micro-block size, 4 in
// the published setting).
//
// A decode query reads every pooled key of its sequence once (128 B each): an HBM
// stream of 2 multiply-adds per byte, too many for the CUDA cores to keep pace
// with HBM once operand conversion and reduction are counted.  The dot products
// therefore run on mma.sync (m16n8k16, bf16 in, fp32 accumulate): 16 blocks x 16
// dims of pooled keys as A, the query's 4 indexer heads (plus 4 zero columns) as
// B, four K-steps per 16 blocks.  Pooled tiles of 128 blocks (16 KiB) stream
// through a 4-slot cp.async ring into XOR-swizzled shared memory (three tiles in
// flight per CTA while the fourth is read, one wave of CTAs); each of the 8 warps
// takes 16 blocks of a tile.  A slot is refilled only after the barrier that
// follows every warp's reads of it.  The epilogue applies ReLU and the head weights with one fp32 FMA chain per block
// (w0*r0, then + w1*r1, + w2*r2, + w3*r3).  fp32 accumulation of bf16 x bf16
// products is exact for small integers.  Optionally the same pass histograms the
// scores' top key digit for the select.

#include <atomic>

#include "select_finish.cuh"

namespace qsa {

namespace {

constexpr int kTile = 128;                       // pooled blocks per stage
constexpr int kStages = 4;                       // ring slots per CTA
constexpr int kTileBytes = kTile * kIdxDim * 2;  // 16 KiB
constexpr int kRingBytes = kStages * kTileBytes;  // 64 KiB
// dynamic shared memory: the copy ring, later (in a row's last CTA) the row's keys
constexpr int kStageBytes = kRingBytes > kRowSmemWords * 4 ? kRingBytes : kRowSmemWords * 4;

__device__ __forceinline__ void cp_async16(uint32_t saddr, const void* g, int src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(saddr), "l"(g), "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

// byte offset of 16-byte chunk `ch` of 128-byte row `row`, XOR-swizzled so that
// 8 consecutive rows at one chunk fall in 8 distinct bank groups
__device__ __forceinline__ uint32_t swz(int row, int ch) { return (uint32_t)(row * 128 + ((ch ^ (row & 7)) << 4)); }

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

}  // namespace

template <bool kHist>
__global__ void __launch_bounds__(256, 2)
k_score_decode(const uint4* __restrict__ q_idx, const float* __restrict__ w, const uint4* __restrict__ pooled,
               const int32_t* __restrict__ q_seq, const int32_t* __restrict__ q_pos, int32_t row0,
               int32_t batch, int64_t kv_capacity, int64_t max_blocks, float* __restrict__ scores,
               int64_t ld, int chunk, TopkCtrl* __restrict__ ctrl, int32_t* __restrict__ sel_idx,
               int32_t* __restrict__ sel_cnt, unsigned* status, int pos_stride, int bs, int top_k)
{
    extern __shared__ __align__(1024) uint8_t s_stage[];
    __shared__ FinishSmem S;  // S.hist: the digit-1 histogram of this CTA's scores
    __shared__ int s_last;
    unsigned* s_hist = S.hist;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int r = blockIdx.y;
    const int i = row0 + r;
    // before griddep_wait: only the layer call's own inputs (rows, query, weights)
    const int s = q_seq[(int64_t)i * pos_stride];
    const int t = q_pos[(int64_t)i * pos_stride];
    const bool ok = (s >= 0 && s < batch && t >= 0 && (int64_t)t < kv_capacity);
    int64_t n_c = ok ? ((int64_t)t + 1) / bs : 0;
    const bool over = n_c > max_blocks;
    if (over) n_c = max_blocks;
    const int64_t b0 = (int64_t)blockIdx.x * chunk;
    const int64_t b_end = min(b0 + (int64_t)chunk, max_blocks);
    const int64_t b_valid = min(b_end, n_c);
    float* srow = scores + (int64_t)r * ld;

    // B operand: column n = lane / 4 is indexer head n (columns 4..7 are zero),
    // rows 2*(lane % 4) (+1, +8, +9) of each 16-dim K-step
    const int g = lane >> 2, c = lane & 3;
    uint32_t bq[4][2];
    {
        const uint32_t* q32 = reinterpret_cast<const uint32_t*>(q_idx) + ((int64_t)i * kIdxHeads + (g & 3)) * 32;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            bq[kk][0] = g < kIdxHeads ? __ldg(q32 + 8 * kk + c) : 0u;
            bq[kk][1] = g < kIdxHeads ? __ldg(q32 + 8 * kk + 4 + c) : 0u;
        }
    }
    const float w0 = __ldg(w + (int64_t)i * kIdxHeads + 0), w1 = __ldg(w + (int64_t)i * kIdxHeads + 1);
    const float w2 = __ldg(w + (int64_t)i * kIdxHeads + 2), w3 = __ldg(w + (int64_t)i * kIdxHeads + 3);
    if (kHist)
        for (int k = tid; k < kBins1; k += 256) s_hist[k] = 0;

    griddep_wait();  // pooled keys, control blocks and the score rows are written from here on
    griddep_launch_dependents();
    if (!ok && blockIdx.x == 0 && tid == 0)
        set_status(status, (s < 0 || s >= batch) ? QSA_DEV_BAD_SEQ : QSA_DEV_BAD_POS);
    if (over && blockIdx.x == 0 && tid == 0) set_status(status, QSA_DEV_BLOCKS_OVER);
    for (int64_t b = max(b0, n_c) + tid; b < b_end; b += 256) srow[b] = -INFINITY;
    if (kHist) __syncthreads();

    if (b0 < b_valid) {
        const uint8_t* prow = reinterpret_cast<const uint8_t*>(pooled) + (int64_t)s * (kv_capacity / bs) * 128;
        const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(s_stage);
        const int n_tiles = (int)((b_valid - b0 + kTile - 1) / kTile);
        // stage tile `tl` into slot tl % kStages: 1,024 chunks of 16 B, 4 per thread
        auto issue = [&](int tl) {
            const uint32_t dst = sbase + (uint32_t)((tl % kStages) * kTileBytes);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int idx = tid + 256 * k;
                const int row = idx >> 3, ch = idx & 7;
                const int64_t b = b0 + (int64_t)tl * kTile + row;
                const bool in = b < b_valid;
                cp_async16(dst + swz(row, ch), prow + (in ? b : 0) * 128 + ch * 16, in ? 16 : 0);
            }
        };
#pragma unroll
        for (int tl = 0; tl < kStages - 1; ++tl) {
            if (tl < n_tiles) issue(tl);
            cp_async_commit();
        }

        const int m = lane >> 3;

        for (int tl = 0; tl < n_tiles; ++tl) {
            // tiles tl .. tl + kStages - 2 are committed: wait for tile tl, then the
            // barrier both publishes every thread's copies of tile tl and ensures every
            // warp has finished reading tile tl - 1, whose slot the next issue reuses
            cp_async_wait<kStages - 2>();
            __syncthreads();
            if (tl + kStages - 1 < n_tiles) issue(tl + kStages - 1);
            cp_async_commit();
            const uint32_t tbase = sbase + (uint32_t)((tl % kStages) * kTileBytes);
            float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                uint32_t a[4];
                ldsm_x4(a, tbase + swz(16 * warp + (lane & 7) + ((m & 1) << 3), 2 * kk + (m >> 1)));
                mma_bf16(d, a, bq[kk][0], bq[kk][1]);
            }
            // lane quad g: lane c = 0 holds heads 0,1 and lane c = 1 heads 2,3 of blocks g and g + 8
            const float r0 = fmaxf(d[0], 0.f), r1 = fmaxf(d[1], 0.f);
            const float r2 = fmaxf(d[2], 0.f), r3 = fmaxf(d[3], 0.f);
            const float u0 = __shfl_down_sync(0xffffffffu, r0, 1), u1 = __shfl_down_sync(0xffffffffu, r1, 1);
            const float u2 = __shfl_down_sync(0xffffffffu, r2, 1), u3 = __shfl_down_sync(0xffffffffu, r3, 1);
            float sa = fmaf(w0, r0, 0.f), sb = fmaf(w0, r2, 0.f);
            sa = fmaf(w1, r1, sa);
            sb = fmaf(w1, r3, sb);
            sa = fmaf(w2, u0, sa);
            sb = fmaf(w2, u2, sb);
            sa = fmaf(w3, u1, sa);
            sb = fmaf(w3, u3, sb);
            const int64_t ba = b0 + (int64_t)tl * kTile + 16 * warp + g;
            const bool ina = c == 0 && ba < b_valid, inb = c == 0 && ba + 8 < b_valid;
            if (ina) srow[ba] = sa;
            if (inb) srow[ba + 8] = sb;
            if (kHist) {
                // one shared-memory atomic per distinct bin per warp
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const bool in = hf ? inb : ina;
                    const unsigned bin = in ? orderable_key(hf ? sb : sa) >> 20 : 0xFFFFFFFFu;
                    const unsigned peers = __match_any_sync(0xffffffffu, bin);
                    if (in && lane == __ffs(peers) - 1) atomicAdd(&s_hist[bin], (unsigned)__popc(peers));
                }
            }
        }
        cp_async_wait<0>();
    }
    if (!kHist) return;

    __syncthreads();
    TopkCtrl* cc = ctrl + r;
    for (int k = tid; k < kBins1; k += 256) {
        const unsigned v = s_hist[k];
        if (v) atomicAdd(&cc->hist1[k], v);
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(&cc->done[0], 1u) == gridDim.x - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (sel_idx) {
        // the row's last CTA selects the whole row in shared memory (n_c <= kRowSmemBlocks)
        select_row_in_smem(S, reinterpret_cast<unsigned*>(s_stage), srow, (int)n_c, top_k, cc->hist1,
                           sel_idx + (int64_t)i * kSelCap, sel_cnt + i);
        return;
    }
    finish_digit1(cc, n_c, top_k, S.warp);
}

cudaError_t launch_score_decode(const qsa_dims& d, const void* q_idx, const float* w, const void* pooled,
                                const int32_t* q_seq, const int32_t* q_pos, int32_t row0, int32_t n_rows,
                                int64_t max_blocks, float* scores, int64_t ld, int chunk, TopkCtrl* ctrl,
                                int32_t* sel_idx, int32_t* sel_cnt, unsigned* status, cudaStream_t st, bool pdl,
                                int pos_stride)
{
    if (sel_idx && (!ctrl || max_blocks > kRowSmemBlocks)) return cudaErrorInvalidValue;
    if (n_rows <= 0 || max_blocks <= 0) return cudaSuccess;
    const int64_t n_chunks = (max_blocks + chunk - 1) / chunk;
    dim3 grid((unsigned)n_chunks, (unsigned)n_rows);
    static std::atomic<bool> attr_set[128];  // per device; setting it twice is harmless
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 128 && !attr_set[dev].load()) {
        cudaError_t e = cudaFuncSetAttribute(k_score_decode<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kStageBytes);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(k_score_decode<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     kStageBytes);
        if (e != cudaSuccess) return e;
        attr_set[dev].store(true);
    }
    return launch_k(ctrl ? k_score_decode<true> : k_score_decode<false>, grid, dim3(256), kStageBytes, st, pdl,
                    (const uint4*)q_idx, w, (const uint4*)pooled, q_seq, q_pos, row0, d.batch, d.kv_capacity,
                    max_blocks, scores, ld, chunk, ctrl, sel_idx, sel_cnt, status, pos_stride, d.block_size, d.top_k);
}

}  // namespace qsa
