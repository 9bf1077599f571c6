// Context parallelism: one long sequence's blocks spread over several GPUs.
//
// The pages say only that several GPUs add memory but add exchange between the
// cards (ai-manual.ru, discussion of llama.cpp PR #30965, closing note).  The
// layer splits exactly along its two reductions:
//   * selection: the global top-k blocks (score descending, lower block index on
//     ties) are a subset of the union of every shard's local top-k, so each GPU
//     selects among its own blocks and ships k 64-bit keys per query
//     (order-preserving score << 32 | ~block); every GPU merges the same union
//     into the same global top-k and keeps the blocks of its own shard;
//   * attention: softmax over a union of token sets is the combination of each
//     set's partial (max, sum of exponentials, exponential-weighted values), so
//     each GPU attends its own selected blocks (and the query's partial block if it
//     holds the query's last tokens) and ships one partial per (query, head).
// The exchanges themselves (two all-gathers) are the caller's (NCCL); these entry
// points are the per-GPU steps between them.  A shard is the block range
// [blk_lo, blk_lo + n_local) of every sequence; the caller's dims describe the
// shard (kv_capacity = n_local * block_size tokens), positions stay global.

#include "select_finish.cuh"

namespace qsa {

namespace {

constexpr int kPartRow = 4 + kHeadDim;  // max, sum, 2 pad, 128 values (floats)

// Global positions -> positions inside the shard: the shard's complete causal blocks
// are n_c(t) - blk_lo clamped to [0, n_local]; a query whose last tokens lie in a
// later shard sees every block of this one and no partial block here; one before the
// shard sees nothing (-1).
__global__ void k_cp_local_pos(const int32_t* __restrict__ q_pos, int32_t n_q, int64_t tok_lo, int64_t cap_loc,
                               int32_t* __restrict__ pos_loc)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n_q) return;
    const int64_t t = q_pos[i];
    int64_t tl = t - tok_lo;
    if (t < 0 || tl < 0) tl = -1;
    else if (tl >= cap_loc) tl = cap_loc - 1;
    pos_loc[i] = (int32_t)tl;
}

// Local selection -> 64-bit keys: order-preserving score in the high word, the
// complement of the global block index in the low word (so a larger key is a higher
// score, then a lower block).  Unused slots are 0 (below every key).
__global__ void __launch_bounds__(256)
k_cp_keys(const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ sel, const int32_t* __restrict__ cnt,
          int64_t blk_lo, unsigned long long* __restrict__ keys, int32_t* __restrict__ key_cnt)
{
    const int i = blockIdx.x;
    const int c = cnt[i];
    for (int j = threadIdx.x; j < kSelCap; j += 256) {
        unsigned long long k = 0ull;
        if (j < c) {
            const int b = sel[(int64_t)i * kSelCap + j];
            const unsigned key = orderable_key(__ldcg(scores + (int64_t)i * ld + b));
            k = ((unsigned long long)key << 32) | (unsigned)(~(uint32_t)(blk_lo + b));
        }
        keys[(int64_t)i * kSelCap + j] = k;
    }
    if (threadIdx.x == 0) key_cnt[i] = c;
}

// One CTA per query: the top_k largest of the shards' keys (at most 8 x 512), then
// the selected blocks in ascending order, globally and restricted to this shard.
__global__ void __launch_bounds__(256)
k_cp_merge(const unsigned long long* __restrict__ keys_all, const int32_t* __restrict__ cnt_all, int n_ranks,
           int32_t n_q, int top_k, int64_t blk_lo, int64_t n_local, int32_t* __restrict__ sel_local,
           int32_t* __restrict__ cnt_local, int32_t* __restrict__ sel_global, int32_t* __restrict__ cnt_global)
{
    __shared__ FinishSmem S;
    __shared__ int s_off[9];
    const int tid = threadIdx.x;
    const int i = blockIdx.x;
    if (tid == 0) {
        s_off[0] = 0;
        for (int r = 0; r < n_ranks; ++r) {
            const int c = cnt_all[(int64_t)r * n_q + i];
            s_off[r + 1] = s_off[r] + (c < 0 ? 0 : c > kSelCap ? kSelCap : c);
        }
        S.n_list = 0;
    }
    for (int k = tid; k < kSelCap; k += 256) S.list[k] = INT_MAX;
    __syncthreads();
    const int nc = s_off[n_ranks];
    // candidates as (score key << 32 | global block), kPerThreadCand per thread
    unsigned long long cr[kPerThreadCand];
#pragma unroll
    for (int k = 0; k < kPerThreadCand; ++k) {
        const int j = tid + 256 * k;
        cr[k] = 0ull;
        if (j < nc) {
            int r = 0;
            while (r + 1 < n_ranks && s_off[r + 1] <= j) ++r;
            const unsigned long long e = keys_all[((int64_t)r * n_q + i) * kSelCap + (j - s_off[r])];
            cr[k] = (e & 0xFFFFFFFF00000000ull) | (unsigned)(~(uint32_t)e);
        }
    }
    const int want = nc < top_k ? nc : top_k;
    if (want > 0) {
        const Cut cut = nc <= top_k ? Cut{0u, 0, true} : resolve_cut_regs(S, cr, nc, top_k, true, 0u);
        // keys equal at the cut come from distinct blocks: the lowest blocks win
        take_by_cut_exact(S, cr, nc, cut);
    }
    __syncthreads();
    sort_list_512(S);
    for (int k = tid; k < kSelCap; k += 256) {
        const int b = k < want ? S.list[k] : -1;
        if (sel_global) sel_global[(int64_t)i * kSelCap + k] = b;
    }
    if (tid == 0 && cnt_global) cnt_global[i] = want;
    // this shard's blocks, still ascending: a prefix count then one pass
    __syncthreads();
    int local_before = 0;
    for (int base = 0; base < want; base += 256) {
        const int k = base + tid;
        const int b = k < want ? S.list[k] : -1;
        const bool mine = k < want && b >= blk_lo && b < blk_lo + n_local;
        int n_mine;
        const int rank = block_rank_256(mine, S.cnt, &n_mine);
        if (mine) sel_local[(int64_t)i * kSelCap + local_before + rank] = (int)(b - blk_lo);
        local_before += n_mine;
    }
    for (int k = local_before + tid; k < kSelCap; k += 256) sel_local[(int64_t)i * kSelCap + k] = -1;
    if (tid == 0) cnt_local[i] = local_before;
}

// out[i][h] = combination of the shards' partials of (query i, head h).
__global__ void __launch_bounds__(128)
k_cp_combine(const float* __restrict__ parts, int n_ranks, int64_t rows, __nv_bfloat16* __restrict__ out)
{
    // 32 threads per row, 4 dims each
    const int64_t row = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
    const int d0 = (threadIdx.x & 31) * 4;
    if (row >= rows) return;
    float Mg = -INFINITY, Lg = 0.f, o[4] = {0.f, 0.f, 0.f, 0.f};
    for (int r = 0; r < n_ranks; ++r) {
        const float* p = parts + ((int64_t)r * rows + row) * kPartRow;
        const float ms = __ldg(p), ls = __ldg(p + 1);
        const float4 v = __ldg(reinterpret_cast<const float4*>(p + 4 + d0));
        const float mn = fmaxf(Mg, ms);
        const float mu = mn == -INFINITY ? 0.f : mn;
        const float fa = exp2f(Mg - mu), fb = exp2f(ms - mu);
        Lg = Lg * fa + ls * fb;
        o[0] = o[0] * fa + v.x * fb;
        o[1] = o[1] * fa + v.y * fb;
        o[2] = o[2] * fa + v.z * fb;
        o[3] = o[3] * fa + v.w * fb;
        Mg = mn;
    }
    const float inv = Lg > 0.f ? 1.f / Lg : 0.f;
    const __nv_bfloat162 a = __floats2bfloat162_rn(o[0] * inv, o[1] * inv);
    const __nv_bfloat162 b = __floats2bfloat162_rn(o[2] * inv, o[3] * inv);
    uint2 w;
    w.x = *reinterpret_cast<const uint32_t*>(&a);
    w.y = *reinterpret_cast<const uint32_t*>(&b);
    *reinterpret_cast<uint2*>(out + row * kHeadDim + d0) = w;
}

}  // namespace

size_t cp_partial_row_floats() { return kPartRow; }

cudaError_t launch_cp_local_pos(const int32_t* q_pos, int32_t n_q, int64_t tok_lo, int64_t cap_loc, int32_t* pos_loc,
                                cudaStream_t st)
{
    if (n_q <= 0) return cudaSuccess;
    k_cp_local_pos<<<(n_q + 255) / 256, 256, 0, st>>>(q_pos, n_q, tok_lo, cap_loc, pos_loc);
    return cudaGetLastError();
}

cudaError_t launch_cp_keys(const float* scores, int64_t ld, const int32_t* sel, const int32_t* cnt, int32_t n_q,
                           int64_t blk_lo, unsigned long long* keys, int32_t* key_cnt, cudaStream_t st)
{
    if (n_q <= 0) return cudaSuccess;
    k_cp_keys<<<n_q, 256, 0, st>>>(scores, ld, sel, cnt, blk_lo, keys, key_cnt);
    return cudaGetLastError();
}

cudaError_t launch_cp_merge(const unsigned long long* keys_all, const int32_t* cnt_all, int n_ranks, int32_t n_q,
                            int top_k, int64_t blk_lo, int64_t n_local, int32_t* sel_local, int32_t* cnt_local,
                            int32_t* sel_global, int32_t* cnt_global, cudaStream_t st)
{
    if (n_q <= 0) return cudaSuccess;
    k_cp_merge<<<n_q, 256, 0, st>>>(keys_all, cnt_all, n_ranks, n_q, top_k, blk_lo, n_local, sel_local, cnt_local,
                                    sel_global, cnt_global);
    return cudaGetLastError();
}

cudaError_t launch_cp_combine(const float* parts, int n_ranks, int64_t rows, void* out, cudaStream_t st)
{
    if (rows <= 0) return cudaSuccess;
    k_cp_combine<<<(unsigned)((rows + 3) / 4), 128, 0, st>>>(parts, n_ranks, rows, (__nv_bfloat16*)out);
    return cudaGetLastError();
}

}  // namespace qsa
