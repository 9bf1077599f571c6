// Micro-block key pooling (step 1 of the QSA layer).
//
// keieiax.jp glossary "Qwen Sparse Attention", section on 4-token micro-blocks:
// the context is compressed into blocks of 4 tokens; blog.cecily.jp/6295
// (Raschka's explainer paragraph): the indexer averages the keys of each block.
// The pooled cache holds one bf16 mean key per complete block and is extended
// as tokens are appended, so each block is pooled exactly once.
//
// HBM-bound and tiny: one thread per (block, 8-dim chunk), one 16-byte load per
// token of the block (4 in the published setting) and one 16-byte store.  The same
// launch clears the layer call's select control blocks and split counters, so
// the decode chain needs no separate memset.

#include "qsa_internal.cuh"

namespace qsa {

__global__ void __launch_bounds__(256)
k_pool_append(const uint4* __restrict__ idx_k, uint4* __restrict__ pooled,
              const int32_t* __restrict__ len_before, const int32_t* __restrict__ len_after,
              int64_t kv_capacity, int bs, int32_t max_new_tokens, int32_t max_new_blocks, int pool_ctas,
              uint4* __restrict__ zero, int64_t zero_words, unsigned* status)
{
    griddep_wait();
    griddep_launch_dependents();
    // side job of the CTAs of row 0: clear the caller's control region
    if (zero && blockIdx.y == 0)
        for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < zero_words; k += (int64_t)gridDim.x * blockDim.x)
            zero[k] = make_uint4(0, 0, 0, 0);
    if ((int)blockIdx.x >= pool_ctas) return;
    const int s = blockIdx.y;
    const int lb = len_before[s];
    const int la = len_after[s];
    if (lb < 0 || la < lb || (int64_t)la > kv_capacity) {
        if (blockIdx.x == 0 && threadIdx.x == 0) set_status(status, QSA_DEV_BAD_LEN);
        return;
    }
    int n = la / bs - lb / bs;
    if (la - lb > max_new_tokens) {
        if (blockIdx.x == 0 && threadIdx.x == 0) set_status(status, QSA_DEV_TOO_MANY_NEW);
        n = min(n, max_new_blocks);
    }
    const int gid = blockIdx.x * blockDim.x + threadIdx.x;
    const int j = gid >> 3;          // which appended block
    const int c = gid & 7;           // which 8-dim chunk of the 64-dim key
    if (j >= n) return;
    const int64_t b = (int64_t)(lb / bs) + j;
    const int64_t nb_cap = kv_capacity / bs;
    // 8 uint4 chunks per 64-dim bf16 row
    const uint4* src = idx_k + ((int64_t)s * kv_capacity + b * bs) * 8 + c;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll 4
    for (int tok = 0; tok < bs; ++tok) {
        const uint4 v = __ldg(src + tok * 8);
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            acc[2 * e] += bf16lo(w4[e]);
            acc[2 * e + 1] += bf16hi(w4[e]);
        }
    }
    // the block size is a power of two: the reciprocal is exact and the mean rounds once
    const float inv = 1.0f / (float)bs;
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const __nv_bfloat16 lo = __float2bfloat16_rn(acc[2 * e] * inv);
        const __nv_bfloat16 hi = __float2bfloat16_rn(acc[2 * e + 1] * inv);
        o[e] = (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
    }
    pooled[((int64_t)s * nb_cap + b) * 8 + c] = make_uint4(o[0], o[1], o[2], o[3]);
}

cudaError_t launch_pool(const qsa_dims& d, const void* idx_k, void* pooled, const int32_t* len_before,
                        const int32_t* len_after, int32_t max_new_tokens, void* zero, size_t zero_bytes,
                        unsigned* status, cudaStream_t st)
{
    const int32_t max_new_blocks = max_new_tokens > 0 ? max_new_tokens / d.block_size + 1 : 0;
    const int pool_ctas = (int)(((int64_t)max_new_blocks * 8 + 255) / 256);
    const int64_t zero_words = zero ? (int64_t)(zero_bytes / 16) : 0;
    const int zero_ctas = (int)((zero_words + 1023) / 1024);  // 4 stores per thread
    const int ctas = pool_ctas > zero_ctas ? pool_ctas : zero_ctas;
    if (ctas == 0) return cudaSuccess;
    return launch_k(k_pool_append, dim3((unsigned)ctas, (unsigned)d.batch), dim3(256), 0, st, false,
                    (const uint4*)idx_k, (uint4*)pooled, len_before, len_after, d.kv_capacity, d.block_size, max_new_tokens,
                    max_new_blocks, pool_ctas, (uint4*)zero, zero_words, status);
}

}  // namespace qsa
