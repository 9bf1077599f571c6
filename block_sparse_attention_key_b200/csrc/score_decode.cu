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
// this is an HBM stream: 4 lanes share a block (16 dims = two 16-byte loads each),
// every thread has 4 blocks (8 loads) in flight, and a 4x4 transpose-reduce over
// the lane quad leaves each lane with the 4 head sums of one block, whose score it
// writes.  fp32 accumulation of bf16 x bf16 products (exact for small integers).
// Optionally the same pass histograms the scores' top key digit for the select.

#include "select_common.cuh"

namespace qsa {

template <bool kHist>
__global__ void __launch_bounds__(256, 2)
k_score_decode(const uint4* __restrict__ q_idx, const float* __restrict__ w, const uint4* __restrict__ pooled,
               const int32_t* __restrict__ q_seq, const int32_t* __restrict__ q_pos, int32_t row0,
               int32_t batch, int64_t kv_capacity, int64_t max_blocks, float* __restrict__ scores,
               int64_t ld, int chunk, TopkCtrl* __restrict__ ctrl, unsigned* status)
{
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

        const uint4* prow = pooled + (int64_t)s * (kv_capacity / kBlock) * 8 + 2 * sub;
        const bool odd = sub & 1, high = sub & 2;

        for (int64_t base = b0; base < b_valid; base += 256) {
            uint4 raw[4][2];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int64_t b = base + grp + 64 * u;
                if (b < b_valid) {
                    raw[u][0] = __ldg(prow + b * 8);
                    raw[u][1] = __ldg(prow + b * 8 + 1);
                } else {
                    raw[u][0] = make_uint4(0, 0, 0, 0);
                    raw[u][1] = make_uint4(0, 0, 0, 0);
                }
            }
            float acc[4][kIdxHeads];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const uint32_t x[8] = {raw[u][0].x, raw[u][0].y, raw[u][0].z, raw[u][0].w,
                                       raw[u][1].x, raw[u][1].y, raw[u][1].z, raw[u][1].w};
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
            const int64_t b = base + grp + 64 * sub;
            if (b < b_valid) {
                srow[b] = score;
                if (kHist) atomicAdd(&s_hist[orderable_key(score) >> 20], 1u);
            }
        }
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
    if (ctrl)
        k_score_decode<true><<<grid, 256, 0, st>>>((const uint4*)q_idx, w, (const uint4*)pooled, q_seq, q_pos,
                                                   row0, d.batch, d.kv_capacity, max_blocks, scores, ld,
                                                   chunk, ctrl, status);
    else
        k_score_decode<false><<<grid, 256, 0, st>>>((const uint4*)q_idx, w, (const uint4*)pooled, q_seq, q_pos,
                                                    row0, d.batch, d.kv_capacity, max_blocks, scores, ld,
                                                    chunk, nullptr, status);
    return cudaGetLastError();
}

}  // namespace qsa
