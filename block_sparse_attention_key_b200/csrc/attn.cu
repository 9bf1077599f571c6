// Gathered GQA attention over the selected blocks (step 4 of the QSA layer).
//
// blog.cecily.jp/6295, trade-off paragraph: a query attends at most 2,048 tokens
// (its selected 4-token blocks) plus the current remainder, i.e. its own partial
// block; every selected block brings all 4 of its tokens.  keieiax.jp glossary
// "Qwen Sparse Attention", speed section: the comparison point is dense GQA, so
// the heads are grouped: query head h reads KV head h / group.
//
// One CTA per (split, KV head, query): the group's query heads (<= 16, one MMA
// M-tile) share one gather.  Selected blocks are 1 KiB contiguous per head in
// the head-major cache; 16 blocks (64 tokens) of K and V per pipeline stage are
// fetched with cp.async into XOR-swizzled shared memory (zero-filled where a
// token is not attended), three stages in flight.  Four warps take 16 tokens of
// a stage each: S = Q K^T and O += P V on mma.sync bf16 tensor cores with fp32
// accumulation, online softmax in the exp2 domain with quad shuffles for the row
// max and sum.  The warps' states merge through shared memory.  Decode calls
// split the block list over up to 8 CTAs (one wave of long CTAs) that form a
// thread-block cluster: the partials meet in the first CTA's shared memory over
// distributed shared memory and it merges them.  (The allocation-free entry point
// keeps the global-memory variant: partials in scratch, the last CTA of a
// (query, KV head) to finish, found by a completion counter, merges them.)

#include <atomic>

#include <cooperative_groups.h>

#include "qsa_internal.cuh"

namespace qsa {

namespace {

constexpr int kTileTok = 64;                     // tokens per stage (64 / block size blocks)
constexpr int kStages = 3;
constexpr int kThreads = 128;
constexpr int kRowBytes = kHeadDim * 2;          // 256 B per token row
constexpr int kStageBytes = kTileTok * kRowBytes; // 16 KiB of K (or V)
constexpr int kMaxSplitBlocks = kSelCap + 1;        // selected blocks + the partial block
constexpr int kMaxClusterSplits = 8;              // splits of one (query, KV head): a portable cluster

constexpr int kSmemQ = 0;
constexpr int kSmemK = kSmemQ + 16 * kRowBytes;
constexpr int kSmemV = kSmemK + kStages * kStageBytes;
constexpr int kSmemValid = kSmemV + kStages * kStageBytes;
constexpr int kSmemBlk = kSmemValid + kStages * kTileTok;
constexpr int kSmemTotal = kSmemBlk + kMaxSplitBlocks * 4 + 60;

__device__ __forceinline__ uint32_t swz(int row, int chunk)
{
    return (uint32_t)(row * kRowBytes + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
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

__device__ __forceinline__ void cp_async16(uint32_t saddr, const void* g, int src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(saddr), "l"(g), "r"(src_bytes));
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }

template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

// Merge the split partials (m, l, o) of one (query, KV head) into its G output
// rows: one pass with a running maximum; the loads of consecutive splits are
// independent.  kDims dims per thread: 8 (G <= 8 rows, 16 threads a row) or 16.
template <int kDims>
__device__ __forceinline__ void merge_splits(const float* __restrict__ base, int n_split, int G,
                                             __nv_bfloat16* __restrict__ out_rows)
{
    constexpr int kTpr = kHeadDim / kDims;  // threads per row
    constexpr int64_t pstride = 16 * 2 + 16 * kHeadDim;
    const int row = threadIdx.x / kTpr, d0 = (threadIdx.x % kTpr) * kDims;
    if (row >= G) return;
    float Mg = -INFINITY, Lg = 0.f, og[kDims];
#pragma unroll
    for (int e = 0; e < kDims; ++e) og[e] = 0.f;
#pragma unroll 8
    for (int sp = 0; sp < n_split; ++sp) {
        const float* ps = base + sp * pstride;
        const float ms = __ldcg(ps + row), ls = __ldcg(ps + 16 + row);
        float4 v[kDims / 4];
#pragma unroll
        for (int e = 0; e < kDims / 4; ++e)
            v[e] = __ldcg(reinterpret_cast<const float4*>(ps + 32 + row * kHeadDim + d0) + e);
        const float mn = fmaxf(Mg, ms);
        const float mu = mn == -INFINITY ? 0.f : mn;
        const float fa = exp2f(Mg - mu), fb = exp2f(ms - mu);
        Lg = Lg * fa + ls * fb;
#pragma unroll
        for (int e = 0; e < kDims / 4; ++e) {
            og[4 * e] = og[4 * e] * fa + v[e].x * fb;
            og[4 * e + 1] = og[4 * e + 1] * fa + v[e].y * fb;
            og[4 * e + 2] = og[4 * e + 2] * fa + v[e].z * fb;
            og[4 * e + 3] = og[4 * e + 3] * fa + v[e].w * fb;
        }
        Mg = mn;
    }
    const float inv = Lg > 0.f ? 1.f / Lg : 0.f;
    uint32_t packed[kDims / 2];
#pragma unroll
    for (int e = 0; e < kDims / 2; ++e) packed[e] = pack_bf16(og[2 * e] * inv, og[2 * e + 1] * inv);
    uint4* dst = reinterpret_cast<uint4*>(out_rows + (int64_t)row * kHeadDim + d0);
#pragma unroll
    for (int e = 0; e < kDims / 8; ++e) dst[e] = make_uint4(packed[4 * e], packed[4 * e + 1], packed[4 * e + 2], packed[4 * e + 3]);
}

// Merge of up to kMaxClusterSplits partials held in this CTA's shared memory
// (pm[split][row], pl[split][row], po[split][row][128]), same arithmetic as merge_splits.
template <int kDims>
__device__ __forceinline__ void merge_cluster(const float* pm, const float* pl, const float* po, int n_split, int G,
                                              __nv_bfloat16* __restrict__ out_rows)
{
    constexpr int kTpr = kHeadDim / kDims;
    const int row = threadIdx.x / kTpr, d0 = (threadIdx.x % kTpr) * kDims;
    if (row >= G) return;
    float Mg = -INFINITY, Lg = 0.f, og[kDims];
#pragma unroll
    for (int e = 0; e < kDims; ++e) og[e] = 0.f;
    for (int sp = 0; sp < n_split; ++sp) {
        const float ms = pm[sp * 16 + row], ls = pl[sp * 16 + row];
        const float mn = fmaxf(Mg, ms);
        const float mu = mn == -INFINITY ? 0.f : mn;
        const float fa = exp2f(Mg - mu), fb = exp2f(ms - mu);
        Lg = Lg * fa + ls * fb;
#pragma unroll
        for (int e = 0; e < kDims; e += 4) {
            const float4 v = *reinterpret_cast<const float4*>(po + (sp * 16 + row) * kHeadDim + d0 + e);
            og[e] = og[e] * fa + v.x * fb;
            og[e + 1] = og[e + 1] * fa + v.y * fb;
            og[e + 2] = og[e + 2] * fa + v.z * fb;
            og[e + 3] = og[e + 3] * fa + v.w * fb;
        }
        Mg = mn;
    }
    const float inv = Lg > 0.f ? 1.f / Lg : 0.f;
    uint32_t packed[kDims / 2];
#pragma unroll
    for (int e = 0; e < kDims / 2; ++e) packed[e] = pack_bf16(og[2 * e] * inv, og[2 * e + 1] * inv);
    uint4* dst = reinterpret_cast<uint4*>(out_rows + (int64_t)row * kHeadDim + d0);
#pragma unroll
    for (int e = 0; e < kDims / 8; ++e) dst[e] = make_uint4(packed[4 * e], packed[4 * e + 1], packed[4 * e + 2], packed[4 * e + 3]);
}

}  // namespace

__global__ void __launch_bounds__(kThreads)
k_sparse_attn(const uint4* __restrict__ q, const uint16_t* __restrict__ k_cache,
              const uint16_t* __restrict__ v_cache, const int32_t* __restrict__ q_seq,
              const int32_t* __restrict__ q_pos, const int32_t* __restrict__ sel_idx,
              const int32_t* __restrict__ sel_cnt, int batch, int n_q_heads, int n_kv_heads,
              int64_t kv_capacity, int bs_log2, int top_k, float scale_log2, int blocks_per_split, int n_split,
              int cluster_merge,
              __nv_bfloat16* __restrict__ out, float* __restrict__ partial, unsigned* __restrict__ counters,
              unsigned* status)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    __shared__ int s_last;
    const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(smem);
    uint8_t* s_valid = smem + kSmemValid;
    int* s_blk = reinterpret_cast<int*>(smem + kSmemBlk);

    const int split = blockIdx.x, g = blockIdx.y, i = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = n_q_heads / n_kv_heads;

    // before griddep_wait: only the layer call's own inputs (row, position, query)
    const int s = q_seq[i];
    const int t = q_pos[i];
    const bool ok = s >= 0 && s < batch && t >= 0 && (int64_t)t < kv_capacity;
    const int bs = 1 << bs_log2;         // tokens per block
    const int ipt = kTileTok >> bs_log2;  // blocks per stage
    const int n_c = ok ? (t + 1) >> bs_log2 : 0;
    const int n_part = ok ? (t + 1) - (n_c << bs_log2) : 0;  // tokens of the partial block
    // query heads of this KV group -> rows 0..G-1 of a 16-row tile, rows >= G zero
    for (int k = tid; k < 16 * 16; k += kThreads) {
        const int row = k >> 4, ch = k & 15;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (row < G && ok) v = __ldg(q + ((int64_t)i * n_q_heads + g * G + row) * 16 + ch);
        *reinterpret_cast<uint4*>(smem + kSmemQ + swz(row, ch)) = v;
    }

    griddep_wait();  // the selection comes from the previous kernel
    griddep_launch_dependents();
    if (!ok && split == 0 && g == 0 && tid == 0)
        set_status(status, (s < 0 || s >= batch) ? QSA_DEV_BAD_SEQ : QSA_DEV_BAD_POS);
    int cnt = ok ? sel_cnt[i] : 0;
    const int cnt_max = n_c < top_k ? n_c : top_k;
    if (cnt < 0 || cnt > cnt_max) {
        if (split == 0 && g == 0 && tid == 0) set_status(status, QSA_DEV_BAD_SEL);
        cnt = cnt < 0 ? 0 : cnt_max;
    }
    const int n_att = cnt + (n_part > 0 ? 1 : 0);
    const int a0 = split * blocks_per_split;
    const int a1 = min(a0 + blocks_per_split, n_att);
    const int n_blk = a1 > a0 ? a1 - a0 : 0;

    for (int k = tid; k < n_blk; k += kThreads) {
        const int a = a0 + k;
        int b = n_c;  // the partial block
        if (a < cnt) {
            b = sel_idx[(int64_t)i * kSelCap + a];
            if (b < 0 || b >= n_c) {
                set_status(status, QSA_DEV_BAD_SEL);
                b = -1;
            }
        }
        s_blk[k] = b;
    }
    __syncthreads();

    const int64_t kv_base = ok ? ((int64_t)s * n_kv_heads + g) * kv_capacity * kHeadDim : 0;
    const int n_tiles = (n_blk + ipt - 1) / ipt;

    auto load_tile = [&](int tile, int stage) {
#pragma unroll
        for (int k = 0; k < (kTileTok * 16) / kThreads; ++k) {
            const int idx = tid + k * kThreads;
            const int row = idx >> 4, ch = idx & 15;
            const int bl = tile * ipt + (row >> bs_log2);
            const int tin = row & (bs - 1);
            const int b = bl < n_blk ? s_blk[bl] : -1;
            const bool valid = b >= 0 && (a0 + bl < cnt || tin < n_part);
            const int64_t off = valid ? kv_base + (((int64_t)b << bs_log2) + tin) * kHeadDim + ch * 8 : 0;
            const uint32_t so = swz(row, ch) + stage * kStageBytes;
            cp_async16(sbase + kSmemK + so, k_cache + off, valid ? 16 : 0);
            cp_async16(sbase + kSmemV + so, v_cache + off, valid ? 16 : 0);
            if (ch == 0) s_valid[stage * kTileTok + row] = valid ? 1 : 0;
        }
    };

#pragma unroll
    for (int st = 0; st < kStages - 1; ++st) {
        if (st < n_tiles) load_tile(st, st);
        cp_async_commit();
    }

    // Q fragments (A operand, 16 rows x 128 dims = 8 k-steps)
    uint32_t qa[8][4];
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
        const int m = lane >> 3;
        ldsm_x4(qa[kk], sbase + kSmemQ + swz((lane & 7) + ((m & 1) << 3), 2 * kk + (m >> 1)));
    }

    float o[16][4];
#pragma unroll
    for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

    for (int tile = 0; tile < n_tiles; ++tile) {
        cp_async_wait<kStages - 2>();
        __syncthreads();
        {
            const int nt = tile + kStages - 1;
            if (nt < n_tiles) load_tile(nt, nt % kStages);
            cp_async_commit();
        }
        const int stage = tile % kStages;
        const uint32_t kbase = sbase + kSmemK + stage * kStageBytes;
        const uint32_t vbase = sbase + kSmemV + stage * kStageBytes;
        const uint8_t* valid = s_valid + stage * kTileTok + 16 * warp;

        float sacc[2][4];
#pragma unroll
        for (int j = 0; j < 2; ++j) sacc[j][0] = sacc[j][1] = sacc[j][2] = sacc[j][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const int m = lane >> 3;
            uint32_t b[4];
            ldsm_x4(b, kbase + swz(16 * warp + (lane & 7) + ((m >> 1) << 3), 2 * kk + (m & 1)));
            mma_bf16(sacc[0], qa[kk], b[0], b[1]);
            mma_bf16(sacc[1], qa[kk], b[2], b[3]);
        }
        float x[2][4];
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int tok = 8 * j + 2 * (lane & 3) + (e & 1);
                x[j][e] = valid[tok] ? sacc[j][e] * scale_log2 : -INFINITY;
            }
        float mx0 = fmaxf(fmaxf(x[0][0], x[0][1]), fmaxf(x[1][0], x[1][1]));
        float mx1 = fmaxf(fmaxf(x[0][2], x[0][3]), fmaxf(x[1][2], x[1][3]));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        const float mu0 = mn0 == -INFINITY ? 0.f : mn0;
        const float mu1 = mn1 == -INFINITY ? 0.f : mn1;
        const float al0 = exp2f(m0 - mu0), al1 = exp2f(m1 - mu1);
        m0 = mn0;
        m1 = mn1;
        float p[2][4];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            p[j][0] = exp2f(x[j][0] - mu0);
            p[j][1] = exp2f(x[j][1] - mu0);
            p[j][2] = exp2f(x[j][2] - mu1);
            p[j][3] = exp2f(x[j][3] - mu1);
        }
        l0 = l0 * al0 + (p[0][0] + p[0][1]) + (p[1][0] + p[1][1]);
        l1 = l1 * al1 + (p[0][2] + p[0][3]) + (p[1][2] + p[1][3]);
#pragma unroll
        for (int n = 0; n < 16; ++n) {
            o[n][0] *= al0;
            o[n][1] *= al0;
            o[n][2] *= al1;
            o[n][3] *= al1;
        }
        uint32_t pa[4];
        pa[0] = pack_bf16(p[0][0], p[0][1]);
        pa[1] = pack_bf16(p[0][2], p[0][3]);
        pa[2] = pack_bf16(p[1][0], p[1][1]);
        pa[3] = pack_bf16(p[1][2], p[1][3]);
#pragma unroll
        for (int nn = 0; nn < 8; ++nn) {
            const int m = lane >> 3;
            uint32_t vb[4];
            ldsm_x4_t(vb, vbase + swz(16 * warp + (lane & 7) + ((m & 1) << 3), 2 * nn + (m >> 1)));
            mma_bf16(o[2 * nn], pa, vb[0], vb[1]);
            mma_bf16(o[2 * nn + 1], pa, vb[2], vb[3]);
        }
    }
    cp_async_wait<0>();
    __syncthreads();

    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);

    // merge the four warps (state in the exp2 domain)
    float* s_o = reinterpret_cast<float*>(smem + kSmemK);            // [4][16][128]
    float* s_m = reinterpret_cast<float*>(smem + kSmemV);            // [4][16]
    float* s_l = s_m + 4 * 16;                                       // [4][16]
    const int r0 = lane >> 2, r1 = r0 + 8;
    if ((lane & 3) == 0) {
        s_m[warp * 16 + r0] = m0;
        s_m[warp * 16 + r1] = m1;
        s_l[warp * 16 + r0] = l0;
        s_l[warp * 16 + r1] = l1;
    }
#pragma unroll
    for (int n = 0; n < 16; ++n) {
        const int d = 8 * n + 2 * (lane & 3);
        *reinterpret_cast<float2*>(s_o + (warp * 16 + r0) * kHeadDim + d) = make_float2(o[n][0], o[n][1]);
        *reinterpret_cast<float2*>(s_o + (warp * 16 + r1) * kHeadDim + d) = make_float2(o[n][2], o[n][3]);
    }
    __syncthreads();

    const int row = tid >> 3;         // 16 rows x 8 threads
    const int d0 = (tid & 7) * 16;    // 16 dims per thread
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, s_m[w * 16 + row]);
    const float Mu = M == -INFINITY ? 0.f : M;
    float L = 0.f, acc[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) acc[e] = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const float f = exp2f(s_m[w * 16 + row] - Mu);
        L += s_l[w * 16 + row] * f;
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[e] += s_o[(w * 16 + row) * kHeadDim + d0 + e] * f;
    }

    if (n_split == 1) {
        if (row < G) {
            const float inv = L > 0.f ? 1.f / L : 0.f;
            uint32_t packed[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) packed[e] = pack_bf16(acc[2 * e] * inv, acc[2 * e + 1] * inv);
            uint4* dst = reinterpret_cast<uint4*>(out + ((int64_t)i * n_q_heads + g * G + row) * kHeadDim + d0);
            dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
            dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
        }
        return;
    }

    if (cluster_merge) {
        // The n_split CTAs of this (query, KV head) form one thread-block cluster: each
        // writes its (m, l, o) into the shared memory of the cluster's first CTA, which
        // merges them.  Every thread of every CTA reaches both cluster barriers.
        namespace cg = cooperative_groups;
        cg::cluster_group cl = cg::this_cluster();
        cl.sync();  // every CTA is past its main loop and warp merge: K/V staging is free
        float* lead = cl.map_shared_rank(reinterpret_cast<float*>(smem + kSmemK), 0);
        float* pm = lead;                    // [kMaxClusterSplits][16]
        float* pl = lead + kMaxClusterSplits * 16;
        float* po = lead + 2 * kMaxClusterSplits * 16;  // [kMaxClusterSplits][16][128]
        if (row < G) {
            if ((tid & 7) == 0) {
                pm[split * 16 + row] = M;
                pl[split * 16 + row] = L;
            }
#pragma unroll
            for (int e = 0; e < 16; e += 4)
                *reinterpret_cast<float4*>(po + (split * 16 + row) * kHeadDim + d0 + e) =
                    make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
        }
        cl.sync();  // all partials are in the first CTA's shared memory
        if (split != 0) return;
        const float* lm = reinterpret_cast<const float*>(smem + kSmemK);
        __nv_bfloat16* orow = out + ((int64_t)i * n_q_heads + g * G) * kHeadDim;
        if (G <= 8) merge_cluster<8>(lm, lm + kMaxClusterSplits * 16, lm + 2 * kMaxClusterSplits * 16, n_split, G, orow);
        else merge_cluster<16>(lm, lm + kMaxClusterSplits * 16, lm + 2 * kMaxClusterSplits * 16, n_split, G, orow);
        return;
    }

    // split-K through global memory: publish this split's (m, l, o), the last split of
    // (i, g) merges all
    const int64_t pair = (int64_t)i * n_kv_heads + g;
    const int64_t pstride = 16 * 2 + 16 * kHeadDim;
    float* pp = partial + (pair * n_split + split) * pstride;
    if (row < G) {
        if ((tid & 7) == 0) {
            pp[row] = M;
            pp[16 + row] = L;
        }
#pragma unroll
        for (int e = 0; e < 16; e += 4)
            *reinterpret_cast<float4*>(pp + 32 + row * kHeadDim + d0 + e) =
                make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(counters + pair, 1u) == (unsigned)n_split - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (G <= 8) merge_splits<8>(partial + pair * n_split * pstride, n_split, G, out + ((int64_t)i * n_q_heads + g * G) * kHeadDim);
    else merge_splits<16>(partial + pair * n_split * pstride, n_split, G, out + ((int64_t)i * n_q_heads + g * G) * kHeadDim);
}

cudaError_t launch_attention(const qsa_dims& d, const void* q, const void* k_cache, const void* v_cache,
                             const int32_t* q_seq, const int32_t* q_pos, const int32_t* sel_idx,
                             const int32_t* sel_cnt, int32_t n_q, void* out, int n_split, float* partial,
                             unsigned* counters, unsigned* status, cudaStream_t st, bool pdl, bool cluster_merge)
{
    if (n_q <= 0) return cudaSuccess;
    if (n_split > kMaxClusterSplits) return cudaErrorInvalidValue;
    int bs_log2 = 0;
    while ((1 << bs_log2) < d.block_size) ++bs_log2;
    const int ipt = kTileTok >> bs_log2;
    const int bps = (kMaxSplitBlocks + n_split - 1) / n_split;
    const int bps_tiles = ((bps + ipt - 1) / ipt) * ipt;
    const float scale = d.softmax_scale > 0.f ? d.softmax_scale : 1.0f / sqrtf((float)d.head_dim);
    const float scale_log2 = scale * 1.4426950408889634f;
    static std::atomic<bool> attr_set[128];  // per device; setting it twice is harmless
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 128 && !attr_set[dev].load()) {
        const cudaError_t e =
            cudaFuncSetAttribute(k_sparse_attn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemTotal);
        if (e != cudaSuccess) return e;
        attr_set[dev].store(true);
    }
    const bool clustered = cluster_merge && n_split > 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)n_split, (unsigned)d.n_kv_heads, (unsigned)n_q);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemTotal;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    if (clustered) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = (unsigned)n_split;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.attrs = na ? attr : nullptr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, k_sparse_attn, (const uint4*)q, (const uint16_t*)k_cache,
                              (const uint16_t*)v_cache, q_seq, q_pos, sel_idx, sel_cnt, d.batch, d.n_q_heads,
                              d.n_kv_heads, d.kv_capacity, bs_log2, d.top_k, scale_log2, bps_tiles, n_split,
                              clustered ? 1 : 0,
                              (__nv_bfloat16*)out, partial, counters, status);
}

}  // namespace qsa
