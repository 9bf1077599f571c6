// Indexer block scores for decode-shaped calls (step 2 of the QSA layer).
//
// blog.cecily.jp/6295 (Raschka's explainer paragraph): a learned indexer rates
// every block from its averaged key; keieiax.jp glossary "Qwen Sparse Attention",
// section on 4-token micro-blocks: the indexer estimates each block's importance.
// The score of block b for query i is
//     sum_h w[i][h] * ReLU( q_idx[i][h] . pooled[s][b] )        (4 heads x 64 dims)
// over the complete causal blocks b < floor((t+1)/4).
//
// A decode query touches every pooled key of its sequence once (128 B each), so
// this is an HBM stream: 4 lanes share a block (16 dims, two 16-byte pieces each).
// Each thread stages its own pieces with cp.async into a private shared-memory
// ring two rounds deep (8 x 16 B per round, 64 KiB in flight per CTA), and a 4x4
// transpose-reduce over the lane quad leaves each lane with the 4 head sums of one
// block, whose score it writes.  fp32 accumulation of bf16 x bf16 products (exact for small integers).
// Optionally the same pass histograms the scores' top key digit for the select.

#include "select_common.cuh"

namespace qsa {

namespace {

constexpr int kRounds = 2;                                 // rounds of 256 blocks in flight per CTA
constexpr int kStageBytes = kRounds * 4 * 2 * 256 * 16;     // 64 KiB of dynamic shared memory

__device__ __forceinline__ void cp_async16(uint32_t saddr, const void* g, int src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(saddr), "l"(g), "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

}  // namespace

template <bool kHist>
__global__ void __launch_bounds__(256, 2)
k_score_decode(const uint4* __restrict__ q_idx, const float* __restrict__ w, const uint4* __restrict__ pooled,
               const int32_t* __restrict__ q_seq, const int32_t* __restrict__ q_pos, int32_t row0,
               int32_t batch, int64_t kv_capacity, int64_t max_blocks, float* __restrict__ scores,
               int64_t ld, int chunk, TopkCtrl* __restrict__ ctrl, unsigned* status)
{
    // per-thread private staging: [round][u][half][thread] x 16 B (conflict-free 16-byte lane stride)
    extern __shared__ __align__(16) uint4 s_stage[];
    __shared__ unsigned s_hist[kHist ? kBins1 : 1];
    __shared__ unsigned s_warp[8];
    __shared__ int s_last;

    const int tid = threadIdx.x;
    const int r = blockIdx.y;
    const int i = row0 + r;
    const int s = q_seq[i];
    const int t = q_pos[i];
    const bool ok = (s >= 0 && s < batch && t >= 0 && (int64_t)t < kv_capacity);
    if (!ok && blockIdx.x == 0 && tid == 0)
        set_status(status, (s < 0 || s >= batch) ? QSA_DEV_BAD_SEQ : QSA_DEV_BAD_POS);
    int64_t n_c = ok ? ((int64_t)t + 1) / kBlock : 0;
    if (n_c > max_blocks) {
        if (blockIdx.x == 0 && tid == 0) set_status(status, QSA_DEV_BLOCKS_OVER);
        n_c = max_blocks;
    }
    const int64_t b0 = (int64_t)blockIdx.x * chunk;
    const int64_t b_end = min(b0 + (int64_t)chunk, max_blocks);
    const int64_t b_valid = min(b_end, n_c);
    float* srow = scores + (int64_t)r * ld;

    for (int64_t b = max(b0, n_c) + tid; b < b_end; b += 256) srow[b] = -INFINITY;
    if (kHist) {
        for (int k = tid; k < kBins1; k += 256) s_hist[k] = 0;
        __syncthreads();
    }

    const int grp = tid >> 2;  // 64 lane quads per CTA
    const int sub = tid & 3;   // this lane's 16-dim slice

    if (b0 < b_valid) {
        const uint4* prow = pooled + (int64_t)s * (kv_capacity / kBlock) * 8 + 2 * sub;
        const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(s_stage);
        const int n_rounds = (int)((b_valid - b0 + 255) / 256);
        // stage round `rd` of this thread's 4 blocks (two 16-byte halves each)
        auto issue = [&](int rd) {
            const int slot = rd % kRounds;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int64_t b = b0 + (int64_t)rd * 256 + grp + 64 * u;
                const bool in = b < b_valid;
                const uint4* src = in ? prow + b * 8 : prow;
#pragma unroll
                for (int hf = 0; hf < 2; ++hf)
                    cp_async16(sbase + (uint32_t)((((slot * 4 + u) * 2 + hf) * 256 + tid) * 16), src + hf,
                               in ? 16 : 0);
            }
        };
#pragma unroll
        for (int rd = 0; rd < kRounds - 1; ++rd) {
            if (rd < n_rounds) issue(rd);
            cp_async_commit();
        }

        float qf[kIdxHeads][16];
#pragma unroll
        for (int h = 0; h < kIdxHeads; ++h) {
            const uint4* src = q_idx + ((int64_t)i * kIdxHeads + h) * 8 + 2 * sub;
            const uint4 a = __ldg(src), c = __ldg(src + 1);
            const uint32_t x[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                qf[h][2 * e] = bf16lo(x[e]);
                qf[h][2 * e + 1] = bf16hi(x[e]);
            }
        }
        float wv[kIdxHeads];
#pragma unroll
        for (int h = 0; h < kIdxHeads; ++h) wv[h] = __ldg(w + (int64_t)i * kIdxHeads + h);
        const bool odd = sub & 1, high = sub & 2;

        for (int rd = 0; rd < n_rounds; ++rd) {
            if (rd + kRounds - 1 < n_rounds) issue(rd + kRounds - 1);
            cp_async_commit();
            cp_async_wait<kRounds - 1>();  // this thread's copies of round rd have landed
            const int slot = rd % kRounds;
            float acc[4][kIdxHeads];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const uint4 lo = s_stage[((slot * 4 + u) * 2 + 0) * 256 + tid];
                const uint4 hi = s_stage[((slot * 4 + u) * 2 + 1) * 256 + tid];
                const uint32_t x[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
                float p[16];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    p[2 * e] = bf16lo(x[e]);
                    p[2 * e + 1] = bf16hi(x[e]);
                }
#pragma unroll
                for (int h = 0; h < kIdxHeads; ++h) {
                    float a = 0.f;
#pragma unroll
                    for (int e = 0; e < 16; ++e) a = fmaf(qf[h][e], p[e], a);
                    acc[u][h] = a;
                }
            }
            // transpose-reduce over the quad: lane `sub` ends with block u = sub, all heads
            float ka[kIdxHeads], kb[kIdxHeads];
#pragma unroll
            for (int h = 0; h < kIdxHeads; ++h) {
                const float send_a = odd ? acc[0][h] : acc[1][h];
                const float send_b = odd ? acc[2][h] : acc[3][h];
                ka[h] = (odd ? acc[1][h] : acc[0][h]) + __shfl_xor_sync(0xffffffffu, send_a, 1);
                kb[h] = (odd ? acc[3][h] : acc[2][h]) + __shfl_xor_sync(0xffffffffu, send_b, 1);
            }
            float score = 0.f;
#pragma unroll
            for (int h = 0; h < kIdxHeads; ++h) {
                const float send = high ? ka[h] : kb[h];
                const float mine = (high ? kb[h] : ka[h]) + __shfl_xor_sync(0xffffffffu, send, 2);
                score = fmaf(wv[h], fmaxf(mine, 0.f), score);
            }
            const int64_t b = b0 + (int64_t)rd * 256 + grp + 64 * sub;
            const bool in = b < b_valid;
            if (in) srow[b] = score;
            if (kHist) {
                // one shared-memory atomic per distinct bin per warp
                const unsigned bin = in ? orderable_key(score) >> 20 : 0xFFFFFFFFu;
                const unsigned peers = __match_any_sync(0xffffffffu, bin);
                if (in && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&s_hist[bin], (unsigned)__popc(peers));
            }
        }
        cp_async_wait<0>();
    }
    if (!kHist) return;

    __syncthreads();
    TopkCtrl* c = ctrl + r;
    for (int k = tid; k < kBins1; k += 256) {
        const unsigned v = s_hist[k];
        if (v) atomicAdd(&c->hist1[k], v);
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(&c->done[0], 1u) == gridDim.x - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    finish_digit1(c, n_c, s_warp);
}

cudaError_t launch_score_decode(const qsa_dims& d, const void* q_idx, const float* w, const void* pooled,
                                const int32_t* q_seq, const int32_t* q_pos, int32_t row0, int32_t n_rows,
                                int64_t max_blocks, float* scores, int64_t ld, int chunk, TopkCtrl* ctrl,
                                unsigned* status, cudaStream_t st)
{
    if (n_rows <= 0 || max_blocks <= 0) return cudaSuccess;
    const int64_t n_chunks = (max_blocks + chunk - 1) / chunk;
    dim3 grid((unsigned)n_chunks, (unsigned)n_rows);
    static bool attr_set[128] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 128 && !attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(k_score_decode<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kStageBytes);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(k_score_decode<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     kStageBytes);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    if (ctrl)
        k_score_decode<true><<<grid, 256, kStageBytes, st>>>((const uint4*)q_idx, w, (const uint4*)pooled, q_seq, q_pos,
                                                   row0, d.batch, d.kv_capacity, max_blocks, scores, ld,
                                                   chunk, ctrl, status);
    else
        k_score_decode<false><<<grid, 256, kStageBytes, st>>>((const uint4*)q_idx, w, (const uint4*)pooled, q_seq, q_pos,
                                                    row0, d.batch, d.kv_capacity, max_blocks, scores, ld,
                                                    chunk, nullptr, status);
    return cudaGetLastError();
}

}  // namespace qsa
