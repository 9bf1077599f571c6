// Gathered GQA attention (step 4 of the QSA layer): every query attends its
// selected blocks and its own partial block; decode steps, multi-token drafts and
// prefill chunks all run this kernel.
//
// blog.cecily.jp/6295, trade-off paragraph: a query attends at most 2,048 tokens
// (its selected 4-token blocks) plus the current remainder; every selected block
// brings its 4 tokens.  keieiax.jp glossary "Qwen Sparse Attention", FAQ: with
// multi-token prediction the selected top blocks are reused across the
// speculative steps, so the k draft queries of a sequence can share one selection
// and one gather ("group" below; a plain decode query is a group of one).  Draft
// query j at position t_j >= t_0 attends the shared blocks (all below t_0) plus
// every token from the selection's first incomplete block up to t_j.
//
// Work unit: one CTA per (split, KV head, group).  Its rows are the group's
// k x G query heads of that KV head (G = query heads per KV head, rows <= 32),
// so the gathered K/V of a block is read once for all of them.  The group's item
// list (selected blocks, then the 1-2 blocks holding the draft tokens' tail) is
// cut into `n_split` contiguous ranges: calls with few (group, KV head) pairs split
// each list over the SMs (one CTA per SM, up to 6 stages in flight); calls with at
// least 148 pairs (prefill chunks, large batches) take one CTA per pair, 3 stages,
// two CTAs per SM, and run every group of KV head 0, then of head 1, ...: a chunk's
// queries pick overlapping blocks (at 128K context each block is picked by about 64
// queries of a 4,096-query chunk), and one head's share of them stays in L2 while
// those queries pass.  Each CTA
//   1. reads its range of the selection with one round of independent loads,
//   2. issues cp.async copies of up to `n_stages` stages (64 tokens of K and of V,
//      32 KiB: 16 blocks of 4 tokens in the published setting) at once into
//      XOR-swizzled shared memory, refilling a slot as soon as it is consumed,
//   3. computes with tokens on the MMA's M side: S^T = K Q^T (16 tokens x 8 rows
//      per mma.sync m16n8k16, fp32 accumulate), an online softmax per row in the
//      exp2 domain (row max over the 8 lanes that share a row, by shuffles), and
//      O^T += V^T P^T, P^T brought from accumulator to operand layout by
//      movmatrix transposes; 4 warps take 16 tokens of a stage each,
//   4. merges its warps through shared memory, then merges the splits either in
//      the first CTA's shared memory over distributed shared memory (the splits
//      of a (group, KV head) form one thread-block cluster) or through global
//      scratch with a last-CTA-to-finish counter.
// Nothing waits on another CTA except the cluster barriers every CTA reaches.

#include <atomic>
#include <climits>
#include <mutex>

#include <cooperative_groups.h>

#include "qsa_internal.cuh"

namespace qsa {

namespace {

constexpr int kTT = 64;                     // tokens per stage (64 / block size blocks)
constexpr int kRow = kHeadDim * 2;          // 256 B per token row
constexpr int kStage = kTT * kRow;          // 16 KiB of K (or of V) per stage
constexpr int kMaxItems = kSelCap + 2;      // selected blocks + up to 2 tail blocks
constexpr int kItemCap = 592;               // items of one split: kMaxItems rounded up to whole stages
constexpr int kSmemQ = 32 * kRow;           // up to 32 rows of queries
constexpr int kDecodeMaxStages = 6;         // 6 x 32 KiB in flight per CTA (one CTA per SM)
constexpr int kDecodeMaxSplits = 16;        // splits of one (group, KV head): one cluster
constexpr int kPairStages = 3;              // stages of a one-CTA-per-pair launch (two CTAs per SM)

__device__ __forceinline__ uint32_t swz(int row, int chunk)
{
    return (uint32_t)(row * kRow + ((chunk ^ (row & 7)) << 4));
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

__device__ __forceinline__ uint32_t movm_t(uint32_t x)
{
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
    return y;
}

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
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
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::); }
__device__ __forceinline__ void cp_wait_pending(int n)
{
    // wait until at most n committed groups are still in flight (n < 8)
    switch (n) {
    case 0: asm volatile("cp.async.wait_group 0;\n" ::); break;
    case 1: asm volatile("cp.async.wait_group 1;\n" ::); break;
    case 2: asm volatile("cp.async.wait_group 2;\n" ::); break;
    case 3: asm volatile("cp.async.wait_group 3;\n" ::); break;
    case 4: asm volatile("cp.async.wait_group 4;\n" ::); break;
    case 5: asm volatile("cp.async.wait_group 5;\n" ::); break;
    case 6: asm volatile("cp.async.wait_group 6;\n" ::); break;
    default: asm volatile("cp.async.wait_group 7;\n" ::); break;
    }
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

// shared-memory offsets for a launch with `stages` stages
struct DecLayout {
    int k, v, tok, ioff, ipos, rowt, total;
};
__host__ __device__ inline DecLayout dec_layout(int stages)
{
    DecLayout L;
    L.k = kSmemQ;
    L.v = L.k + stages * kStage;
    L.tok = L.v + stages * kStage;
    L.ioff = L.tok + stages * kTT * 4;
    L.ipos = L.ioff + kItemCap * 8;
    L.rowt = L.ipos + kItemCap * 4;
    L.total = L.rowt + 32 * 4 + 64;
    return L;
}

// per-(pair, split) slot of global partials: m[32], l[32], o[32][128]
constexpr int64_t kPartStride = 64 + 32 * kHeadDim;
constexpr int kMaxPartialSlots = 148;
constexpr int kPartRow = 4 + kHeadDim;       // shard partial of one (query, head): max, sum, pad, values

}  // namespace

// NT = 8-row column tiles of the MMA's N side (rows = k x G <= 8 * NT); NWG = groups
// of 4 compute warps, each group taking every NWG-th stage with its own softmax state.
template <int NT, int NWG>
__global__ void __launch_bounds__(128 * NWG)
k_sparse_attn(const uint4* __restrict__ q, const uint16_t* __restrict__ k_cache, const uint16_t* __restrict__ v_cache,
              const int32_t* __restrict__ q_seq, const int32_t* __restrict__ q_pos,
              const int32_t* __restrict__ sel_idx, const int32_t* __restrict__ sel_cnt,
              const int32_t* __restrict__ page_table, int page_tokens, int64_t table_ld, int64_t n_pages,
              int batch, int n_q_heads, int n_kv_heads, int64_t kv_capacity, int bs_log2, int top_k, int group_q,
              float scale_log2, int items_per_split, int n_split, int n_stages, int merge, int grp_fast,
              __nv_bfloat16* __restrict__ out, float* __restrict__ part_out,
              float* __restrict__ partial, unsigned* __restrict__ counters, unsigned* status)
{
    constexpr int RP = 8 * NT;           // padded rows
    constexpr int kT = 128 * NWG;        // threads
    constexpr int kW = 4 * NWG;          // warps
    constexpr int kPerT = (kItemCap + kT - 1) / kT;
    extern __shared__ __align__(1024) uint8_t smem[];
    __shared__ int s_cnt, s_nitems, s_last, s_seq, s_nc0, s_tlast;
    const DecLayout SL = dec_layout(n_stages);
    const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(smem);
    int* s_tok = reinterpret_cast<int*>(smem + SL.tok);
    long long* s_ioff = reinterpret_cast<long long*>(smem + SL.ioff);
    int* s_ipos = reinterpret_cast<int*>(smem + SL.ipos);
    int* s_rowt = reinterpret_cast<int*>(smem + SL.rowt);

    // grid (splits, KV heads, groups), or (groups, KV heads) for one CTA per pair
    const int split = grp_fast ? 0 : blockIdx.x, g = blockIdx.y, grp = grp_fast ? blockIdx.x : blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = n_q_heads / n_kv_heads;
    const int R = group_q * G;
    const int64_t qi0 = (int64_t)grp * group_q;
    const int bs = 1 << bs_log2;     // tokens per block
    const int ipt = kTT >> bs_log2;  // blocks per stage

    // ---- before griddep_wait: the call's own inputs, one round of independent loads ----
    if (warp == 0) {
        // lane r < RP: row r = (draft query j = r / G, head r % G); its position, or -2
        const int s0 = q_seq[qi0], t0 = q_pos[qi0];
        const bool ok0 = s0 >= 0 && s0 < batch && t0 >= 0 && (int64_t)t0 < kv_capacity;
        const int nc0 = ok0 ? (t0 + 1) >> bs_log2 : 0;
        int t = -2;
        if (lane < R && ok0) {
            const int j = lane / G;
            const int sj = q_seq[qi0 + j], tj = q_pos[qi0 + j];
            // a draft query follows the selection's query within the two tail blocks
            const bool ok = sj == s0 && tj >= t0 && tj <= bs * nc0 + 2 * bs - 1 && (int64_t)tj < kv_capacity;
            if (ok) t = tj;
            else if (split == 0 && g == 0 && lane % G == 0)
                set_status(status, sj != s0 ? QSA_DEV_BAD_SEQ : QSA_DEV_BAD_POS);
        }
        if (lane < RP) s_rowt[lane] = t;
        const int tl = __reduce_max_sync(0xffffffffu, lane < R ? t : -2);
        if (lane == 0) {
            s_seq = ok0 ? s0 : -1;
            s_nc0 = nc0;
            s_tlast = tl;
            if (!ok0 && split == 0 && g == 0)
                set_status(status, (s0 < 0 || s0 >= batch) ? QSA_DEV_BAD_SEQ : QSA_DEV_BAD_POS);
        }
    }
    // query rows (rows of invalid queries attend nothing, so their values do not matter)
    for (int k = tid; k < RP * 16; k += kT) {
        const int row = k >> 4, ch = k & 15;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (row < R) v = __ldg(q + ((qi0 + row / G) * n_q_heads + (int64_t)g * G + row % G) * 16 + ch);
        *reinterpret_cast<uint4*>(smem + swz(row, ch)) = v;
    }

    griddep_wait();  // the selection comes from the previous kernel
    griddep_launch_dependents();

    // ---- this split's items: one round of independent loads ----
    const int a0 = split * items_per_split;
    int raw[kPerT];
#pragma unroll
    for (int u = 0; u < kPerT; ++u) {
        const int k = tid + u * kT;
        const int a = a0 + k;
        raw[u] = (k < items_per_split && a < kSelCap) ? __ldg(sel_idx + (int64_t)grp * kSelCap + a) : -1;
    }
    const int cnt_raw = tid == 0 ? sel_cnt[grp] : 0;
    __syncthreads();  // s_seq, s_nc0, s_tlast, s_rowt, query rows
    if (tid == 0) {
        int cnt = s_seq >= 0 ? cnt_raw : 0;
        const int cnt_max = min(s_nc0, top_k);
        if (cnt < 0 || cnt > cnt_max) {
            if (split == 0 && g == 0) set_status(status, QSA_DEV_BAD_SEL);
            cnt = cnt < 0 ? 0 : cnt_max;
        }
        const int tl = s_tlast;
        const int tail0 = bs * s_nc0;
        const int n_tail = tl >= tail0 ? ((tl - tail0) >> bs_log2) + 1 : 0;
        s_cnt = cnt;
        s_nitems = cnt + n_tail;
    }
    __syncthreads();
    const int cnt = s_cnt;
    const int n_blk = max(0, min(a0 + items_per_split, s_nitems) - a0);
    const int s = s_seq;
    const int nc0 = s_nc0;
#pragma unroll
    for (int u = 0; u < kPerT; ++u) {
        const int k = tid + u * kT;
        if (k >= n_blk) continue;
        const int a = a0 + k;
        int p0 = -1, ipos = -1;  // first token of the item; ipos -1: visible to every row
        if (a < cnt) {
            const int b = raw[u];
            if (b >= 0 && b < nc0) p0 = b << bs_log2;
            else set_status(status, QSA_DEV_BAD_SEL);
        } else {
            p0 = (nc0 + (a - cnt)) << bs_log2;
            ipos = p0;
        }
        long long off = -1;
        if (p0 >= 0) {
            if (page_table) {
                const int page = __ldg(page_table + (int64_t)s * table_ld + p0 / page_tokens);
                if (page >= 0 && page < n_pages)
                    off = (((long long)page * n_kv_heads + g) * page_tokens + p0 % page_tokens) * kHeadDim;
                else
                    set_status(status, QSA_DEV_BAD_PAGE);
            } else {
                off = (((long long)s * n_kv_heads + g) * kv_capacity + p0) * kHeadDim;
            }
        }
        s_ioff[k] = off;
        s_ipos[k] = ipos;
    }
    __syncthreads();

    const int tlast = s_tlast;
    const int n_tiles = (n_blk + ipt - 1) / ipt;
    // four threads per token row, each copying chunks q, q + 4, q + 8, q + 12 (16 B each):
    // one row lookup per thread and tile, 64 contiguous bytes per row per copy instruction
    constexpr int kRowsPerPass = kT / 4;
    auto load_tile = [&](int tile, int slot) {
        const int q4 = tid & 3;
#pragma unroll
        for (int u = 0; u < kTT / kRowsPerPass; ++u) {
            const int row = (tid >> 2) + u * kRowsPerPass;
            const int it = tile * ipt + (row >> bs_log2);
            const int tin = row & (bs - 1);
            long long off = -1;
            int tp = INT_MAX;
            if (it < n_blk) {
                off = s_ioff[it];
                const int ip = s_ipos[it];
                if (off >= 0 && ip >= 0 && ip + tin > tlast) off = -1;  // past the group's last draft token
                if (off >= 0) tp = ip < 0 ? -1 : ip + tin;
            }
            const bool valid = off >= 0;
            const long long e = valid ? off + (long long)tin * kHeadDim : 0;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int ch = q4 + 4 * k;
                const uint32_t so = swz(row, ch) + slot * kStage;
                cp_async16(sbase + SL.k + so, k_cache + e + (valid ? ch * 8 : 0), valid ? 16 : 0);
                cp_async16(sbase + SL.v + so, v_cache + e + (valid ? ch * 8 : 0), valid ? 16 : 0);
            }
            if (q4 == 0) s_tok[slot * kTT + row] = tp;
        }
    };

    // every slot is filled at once; later tiles refill the slots of a finished round
    int issued = 0;
    for (; issued < n_stages && issued < n_tiles; ++issued) {
        load_tile(issued, issued);
        cp_commit();
    }

    const int wg = warp >> 2;        // compute group
    const int wq = warp & 3;         // warp within the group: 16 tokens of the stage
    const int c4 = lane & 3, l4 = lane >> 2;
    int trow[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        trow[nt][0] = s_rowt[8 * nt + 2 * c4];
        trow[nt][1] = s_rowt[8 * nt + 2 * c4 + 1];
    }
    // Q^T fragments (B operand: k = dims, n = rows), held in registers for NT <= 2
    constexpr bool kHoldQ = NT <= 2;
    uint32_t qb[kHoldQ ? 8 : 1][NT][2];
    auto load_qb = [&](int kk2, uint32_t (&dst)[2][NT][2]) {
        // dims of k-steps kk2, kk2 + 1 for every column tile
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            uint32_t r[4];
            ldsm_x4(r, sbase + swz(8 * nt + (lane & 7), 2 * kk2 + (lane >> 3)));
            dst[0][nt][0] = r[0];
            dst[0][nt][1] = r[1];
            dst[1][nt][0] = r[2];
            dst[1][nt][1] = r[3];
        }
    };
    if constexpr (kHoldQ) {
#pragma unroll
        for (int kk = 0; kk < 8; kk += 2) {
            uint32_t t2[2][NT][2];
            load_qb(kk, t2);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                qb[kk][nt][0] = t2[0][nt][0];
                qb[kk][nt][1] = t2[0][nt][1];
                qb[kk + 1][nt][0] = t2[1][nt][0];
                qb[kk + 1][nt][1] = t2[1][nt][1];
            }
        }
    }

    float o[8][NT][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) o[mt][nt][0] = o[mt][nt][1] = o[mt][nt][2] = o[mt][nt][3] = 0.f;
    float m[NT][2], l[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) m[nt][0] = m[nt][1] = -INFINITY, l[nt][0] = l[nt][1] = 0.f;

    for (int r0 = 0; r0 < n_tiles; r0 += NWG) {
        // tiles r0 .. r0 + NWG - 1 have landed (this thread's copies), then every thread's
        const int done = min(n_tiles, r0 + NWG);
        cp_wait_pending(issued - done);
        __syncthreads();
        const int tile = r0 + wg;
        const int slot = tile % n_stages;
        const uint32_t kb = sbase + SL.k + slot * kStage;
        const uint32_t vb = sbase + SL.v + slot * kStage;
        const int tok0 = 16 * wq;
        const bool have = tile < n_tiles;
        const int tp0 = have ? s_tok[slot * kTT + tok0 + l4] : INT_MAX;
        const int tp1 = have ? s_tok[slot * kTT + tok0 + l4 + 8] : INT_MAX;

        if (__any_sync(0xffffffffu, tp0 != INT_MAX || tp1 != INT_MAX)) {  // skip a warp's empty tokens
            // S^T = K Q^T over 128 dims: two independent accumulator chains (even / odd k-steps)
            float sa[NT][4], sb[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) sa[nt][e] = sb[nt][e] = 0.f;
#pragma unroll
            for (int kk = 0; kk < 8; kk += 2) {
                uint32_t ka[4], kb2[4];
                ldsm_x4(ka, kb + swz(tok0 + (lane & 7) + (((lane >> 3) & 1) << 3), 2 * kk + (lane >> 4)));
                ldsm_x4(kb2, kb + swz(tok0 + (lane & 7) + (((lane >> 3) & 1) << 3), 2 * (kk + 1) + (lane >> 4)));
                if constexpr (kHoldQ) {
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        mma16816(sa[nt], ka, qb[kk][nt][0], qb[kk][nt][1]);
                        mma16816(sb[nt], kb2, qb[kk + 1][nt][0], qb[kk + 1][nt][1]);
                    }
                } else {
                    uint32_t t2[2][NT][2];
                    load_qb(kk, t2);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        mma16816(sa[nt], ka, t2[0][nt][0], t2[0][nt][1]);
                        mma16816(sb[nt], kb2, t2[1][nt][0], t2[1][nt][1]);
                    }
                }
            }
            uint32_t pb[NT][2];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                // element e: token l4 (+8 for e >= 2), row 8nt + 2c4 + (e & 1)
                float x[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int tp = e < 2 ? tp0 : tp1;
                    x[e] = tp <= trow[nt][e & 1] ? (sa[nt][e] + sb[nt][e]) * scale_log2 : -INFINITY;
                }
                float a[2];
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    float mx = fmaxf(x[j], x[j + 2]);
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                    const float mn = fmaxf(m[nt][j], mx);
                    const float mu = mn == -INFINITY ? 0.f : mn;
                    a[j] = exp2f(m[nt][j] - mu);
                    const float p0 = exp2f(x[j] - mu), p1 = exp2f(x[j + 2] - mu);
                    x[j] = p0;
                    x[j + 2] = p1;
                    l[nt][j] = l[nt][j] * a[j] + (p0 + p1);
                    m[nt][j] = mn;
                }
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    o[mt][nt][0] *= a[0];
                    o[mt][nt][1] *= a[1];
                    o[mt][nt][2] *= a[0];
                    o[mt][nt][3] *= a[1];
                }
                pb[nt][0] = movm_t(pack_bf16(x[0], x[1]));  // tokens 0-7 -> B operand (k = token, n = row)
                pb[nt][1] = movm_t(pack_bf16(x[2], x[3]));  // tokens 8-15
            }
            // O^T += V^T P^T: 8 tiles of 16 dims
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                uint32_t va[4];
                ldsm_x4_t(va, vb + swz(tok0 + (lane & 7) + ((lane >> 4) << 3), 2 * mt + ((lane >> 3) & 1)));
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma16816(o[mt][nt], va, pb[nt][0], pb[nt][1]);
            }
        }
        __syncthreads();  // every warp is done with this round's slots
        for (int u = 0; u < NWG && issued < n_tiles; ++u) {
            load_tile(issued, issued % n_stages);
            cp_commit();
            ++issued;
        }
    }
    cp_wait_pending(0);
    __syncthreads();

    // ---- merge the warps: (m, l) per row, O^T into shared memory (stage area) ----
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            l[nt][j] += __shfl_xor_sync(0xffffffffu, l[nt][j], 4);
            l[nt][j] += __shfl_xor_sync(0xffffffffu, l[nt][j], 8);
            l[nt][j] += __shfl_xor_sync(0xffffffffu, l[nt][j], 16);
        }
    float* s_o = reinterpret_cast<float*>(smem + SL.k);  // [kW][RP][128]
    float* s_m = s_o + kW * RP * kHeadDim;                // [kW][RP]
    float* s_l = s_m + kW * RP;                           // [kW][RP]
    if (l4 == 0) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                s_m[warp * RP + 8 * nt + 2 * c4 + j] = m[nt][j];
                s_l[warp * RP + 8 * nt + 2 * c4 + j] = l[nt][j];
            }
    }
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int row = 8 * nt + 2 * c4 + (e & 1);
                const int d = 16 * mt + l4 + ((e >> 1) << 3);
                s_o[(warp * RP + row) * kHeadDim + d] = o[mt][nt][e];
            }
    __syncthreads();

    constexpr int TPR = kT / RP;          // threads per row
    constexpr int DPT = kHeadDim / TPR;   // dims per thread: 4 .. 32
    const int row = tid / TPR, d0 = (tid % TPR) * DPT;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kW; ++w) M = fmaxf(M, s_m[w * RP + row]);
    const float Mu = M == -INFINITY ? 0.f : M;
    float L = 0.f, acc[DPT];
#pragma unroll
    for (int e = 0; e < DPT; ++e) acc[e] = 0.f;
#pragma unroll
    for (int w = 0; w < kW; ++w) {
        const float f = exp2f(s_m[w * RP + row] - Mu);
        L += s_l[w * RP + row] * f;
#pragma unroll
        for (int e = 0; e < DPT; ++e) acc[e] += s_o[(w * RP + row) * kHeadDim + d0 + e] * f;
    }
    const bool live_row = row < R;
    __nv_bfloat16* orow = live_row
        ? out + ((qi0 + row / G) * n_q_heads + (int64_t)g * G + row % G) * kHeadDim + d0 : nullptr;

    auto store = [&](float Mg, float Lg, const float* og) {
        if (part_out) {
            // unnormalised partial of a context shard: (max, sum, weighted values), exp2 domain
            float* pr = part_out + ((qi0 + row / G) * n_q_heads + (int64_t)g * G + row % G) * kPartRow;
            if (d0 == 0) {
                pr[0] = Mg;
                pr[1] = Lg;
            }
#pragma unroll
            for (int e = 0; e < DPT; e += 4)
                *reinterpret_cast<float4*>(pr + 4 + d0 + e) = make_float4(og[e], og[e + 1], og[e + 2], og[e + 3]);
            return;
        }
        const float inv = Lg > 0.f ? 1.f / Lg : 0.f;
#pragma unroll
        for (int e = 0; e < DPT; e += 4) {
            uint2 v;
            v.x = pack_bf16(og[e] * inv, og[e + 1] * inv);
            v.y = pack_bf16(og[e + 2] * inv, og[e + 3] * inv);
            *reinterpret_cast<uint2*>(orow + e) = v;
        }
    };
    auto combine = [&](float& Mg, float& Lg, float* og, float ms, float ls, const float* po) {
        const float mn = fmaxf(Mg, ms);
        const float mu = mn == -INFINITY ? 0.f : mn;
        const float fa = exp2f(Mg - mu), fb = exp2f(ms - mu);
        Lg = Lg * fa + ls * fb;
#pragma unroll
        for (int e = 0; e < DPT; e += 4) {
            const float4 v = *reinterpret_cast<const float4*>(po + e);
            og[e] = og[e] * fa + v.x * fb;
            og[e + 1] = og[e + 1] * fa + v.y * fb;
            og[e + 2] = og[e + 2] * fa + v.z * fb;
            og[e + 3] = og[e + 3] * fa + v.w * fb;
        }
        Mg = mn;
    };

    if (n_split == 1) {
        if (live_row) store(M, L, acc);
        return;
    }

    if (merge == 1) {
        // the n_split CTAs of this (group, KV head) form one cluster: partials meet in
        // the first CTA's shared memory; every thread of every CTA reaches both barriers
        namespace cg = cooperative_groups;
        cg::cluster_group cl = cg::this_cluster();
        cl.sync();  // every CTA has finished its warp merge: stage areas are free
        float* lead = cl.map_shared_rank(reinterpret_cast<float*>(smem + SL.k), 0);
        float* po = lead;                                       // [n_split][RP][128]
        float* pm = lead + (size_t)n_split * RP * kHeadDim;     // [n_split][RP]
        float* pl = pm + n_split * RP;                          // [n_split][RP]
        if ((tid % TPR) == 0) {
            pm[split * RP + row] = M;
            pl[split * RP + row] = L;
        }
#pragma unroll
        for (int e = 0; e < DPT; e += 4)
            *reinterpret_cast<float4*>(po + (split * RP + row) * kHeadDim + d0 + e) =
                make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
        cl.sync();
        if (split != 0 || !live_row) return;
        const float* lpo = reinterpret_cast<const float*>(smem + SL.k);
        const float* lpm = lpo + (size_t)n_split * RP * kHeadDim;
        const float* lpl = lpm + n_split * RP;
        float Mg = -INFINITY, Lg = 0.f, og[DPT];
#pragma unroll
        for (int e = 0; e < DPT; ++e) og[e] = 0.f;
        for (int sp = 0; sp < n_split; ++sp)
            combine(Mg, Lg, og, lpm[sp * RP + row], lpl[sp * RP + row], lpo + (sp * RP + row) * kHeadDim + d0);
        store(Mg, Lg, og);
        return;
    }

    // global scratch: publish this split's partial; the last split of the pair merges
    const int64_t pair = (int64_t)grp * n_kv_heads + g;
    float* pp = partial + (pair * n_split + split) * kPartStride;
    if ((tid % TPR) == 0) {
        pp[row] = M;
        pp[32 + row] = L;
    }
#pragma unroll
    for (int e = 0; e < DPT; e += 4)
        *reinterpret_cast<float4*>(pp + 64 + row * kHeadDim + d0 + e) = make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(counters + pair, 1u) == (unsigned)n_split - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (tid == 0) counters[pair] = 0u;  // every split has arrived: ready for the next call
    if (!live_row) return;
    // this split's own partial is still in registers; the others from L2, all loads at once
    const float* base = partial + pair * n_split * kPartStride;
    float Mg = -INFINITY, Lg = 0.f, og[DPT];
#pragma unroll
    for (int e = 0; e < DPT; ++e) og[e] = 0.f;
    for (int sp = 0; sp < n_split; ++sp) {
        const float* ps = base + sp * kPartStride;
        float po[DPT];
        float ms, ls;
        if (sp == split) {
            ms = M;
            ls = L;
#pragma unroll
            for (int e = 0; e < DPT; ++e) po[e] = acc[e];
        } else {
            ms = __ldcg(ps + row);
            ls = __ldcg(ps + 32 + row);
#pragma unroll
            for (int e = 0; e < DPT; e += 4) {
                const float4 v = __ldcg(reinterpret_cast<const float4*>(ps + 64 + row * kHeadDim + d0 + e));
                po[e] = v.x;
                po[e + 1] = v.y;
                po[e + 2] = v.z;
                po[e + 3] = v.w;
            }
        }
        combine(Mg, Lg, og, ms, ls, po);
    }
    store(Mg, Lg, og);
}

// ---------------------------------------------------------------- host side

namespace {

int nt_for_rows(int rows) { return rows <= 8 ? 1 : rows <= 16 ? 2 : 4; }
// compute groups: two for up to 16 rows; one for 32 (its accumulators fill the registers)
int nwg_for(int nt) { return nt <= 2 ? 2 : 1; }

const void* kernel_for(int nt)
{
    return nt == 1 ? (const void*)k_sparse_attn<1, 2> : nt == 2 ? (const void*)k_sparse_attn<2, 2>
                                                                : (const void*)k_sparse_attn<4, 1>;
}

// cluster-merge buffer in the lead CTA's stage area: partials of n_split CTAs, rp rows each
int merge_bytes(int n_split, int rp) { return n_split * rp * (kHeadDim + 2) * 4; }

struct Plan {
    int n_split, stages, ips, smem;
    bool cluster;
};

// How many clusters of `n_split` CTAs with `smem` bytes each the device can hold
// at once (cached per device and shape).
int active_clusters(int dev, int nt, int n_split, int smem)
{
    static std::mutex mu;
    static int cache[64][3][17][8];  // [dev][nt index][n_split][stages-1], 0 = unknown, -1 = none
    const int ni = nt == 1 ? 0 : nt == 2 ? 1 : 2;
    const int si = (smem - dec_layout(1).total) / (2 * kStage);
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= 64 || n_split > 16 || si < 0 || si >= 8) return 0;
    int& c = cache[dev][ni][n_split][si];
    if (c == 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)n_split, 1, 1);
        cfg.blockDim = dim3(128 * nwg_for(nt));
        cfg.dynamicSmemBytes = (size_t)smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)n_split;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kernel_for(nt), &cfg) != cudaSuccess) {
            cudaGetLastError();
            n = 0;
        }
        c = n > 0 ? n : -1;
    }
    return c > 0 ? c : 0;
}

bool configure(int dev, int nt)
{
    static std::atomic<bool> done[64][3];
    const int ni = nt == 1 ? 0 : nt == 2 ? 1 : 2;
    if (dev < 0 || dev >= 64) return false;
    if (done[dev][ni].load()) return true;
    const void* fn = kernel_for(nt);
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, dec_layout(kDecodeMaxStages).total) !=
            cudaSuccess ||
        cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
        return false;
    done[dev][ni].store(true);
    return true;
}

// Splits of a (group, KV head) pair's item list: as many as keep one CTA on every SM
// (each streams its whole share with every stage in flight).  The splits merge in a
// cluster when the device can hold every cluster at once, else through global scratch.
Plan plan(int dev, int64_t pairs, int rows, bool allow_cluster, int ipt)
{
    const int nt = nt_for_rows(rows);
    const int rp = 8 * nt;
    const int warps = 4 * nwg_for(nt);
    const int tiles_max = (kMaxItems + ipt - 1) / ipt;  // 33 stages of 16 blocks of 4 tokens
    for (int ns = attn_split_bound(pairs); ns >= 1; --ns) {
        const int tiles = (tiles_max + ns - 1) / ns;
        int stages = tiles < kDecodeMaxStages ? tiles : kDecodeMaxStages;
        if (stages < 2 * nwg_for(nt) && tiles > stages) stages = 2 * nwg_for(nt);
        // the warp merge (and the cluster merge) buffers live in the stage area
        const int warp_merge = warps * rp * (kHeadDim + 2) * 4;
        while (stages * 2 * kStage < warp_merge) ++stages;
        bool cluster = false;
        if (ns > 1 && allow_cluster) {
            int cs = stages;
            while (cs * 2 * kStage < merge_bytes(ns, rp)) ++cs;
            if (cs <= kDecodeMaxStages && (int64_t)active_clusters(dev, nt, ns, dec_layout(cs).total) >= pairs) {
                cluster = true;
                stages = cs;
            }
        }
        if (stages > kDecodeMaxStages) continue;  // too many rows for this many splits
        if (ns == 1 && pairs >= 148 && stages > kPairStages && warp_merge <= kPairStages * 2 * kStage)
            stages = kPairStages;  // one CTA per pair: two CTAs per SM
        return Plan{ns, stages, tiles * ipt, dec_layout(stages).total, cluster};
    }
    return Plan{1, kDecodeMaxStages, tiles_max * ipt, dec_layout(kDecodeMaxStages).total, false};
}

}  // namespace

bool describe_sparse_attn(const qsa_dims& d, int64_t n_groups, int group_q, bool allow_cluster, int* n_split,
                          int* stages, int* threads, int* smem, int64_t* ctas, int* cluster, int* rows)
{
    const int G = d.n_q_heads / d.n_kv_heads;
    const int r = G * group_q;
    if (r > 32 || n_groups <= 0) return false;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || !configure(dev, nt_for_rows(r))) {
        // no device: the plan without the occupancy query of the cluster merge
        cudaGetLastError();
        dev = 0;
        allow_cluster = false;
    }
    int bs_log2 = 0;
    while ((1 << bs_log2) < d.block_size) ++bs_log2;
    const int64_t pairs = n_groups * d.n_kv_heads;
    const Plan p = plan(dev, pairs, r, allow_cluster, kTT >> bs_log2);
    *n_split = p.n_split;
    *stages = p.stages;
    *threads = 128 * nwg_for(nt_for_rows(r));
    *smem = p.smem;
    *ctas = pairs * p.n_split;
    *cluster = p.cluster ? 1 : 0;
    *rows = r;
    return true;
}

int attn_split_bound(int64_t pairs)
{
    if (pairs <= 0 || pairs >= 148) return 1;
    const int64_t want = 148 / pairs;
    return (int)(want > kDecodeMaxSplits ? kDecodeMaxSplits : want);
}

size_t attn_counter_bytes()
{
    // only split launches count arrivals, and they have fewer than 148 pairs
    return (size_t)kMaxPartialSlots * 4;
}

size_t attn_partial_bytes()
{
    // a launch splits only when (groups x KV heads) < 148, into at most
    // min(16, 148 / pairs) splits: at most 148 (pair, split) slots
    return (size_t)kMaxPartialSlots * kPartStride * 4;
}

cudaError_t launch_sparse_attn(const qsa_dims& d, const void* q, const void* k_cache, const void* v_cache,
                               const int32_t* q_seq, const int32_t* q_pos, const int32_t* sel_idx,
                               const int32_t* sel_cnt, const int32_t* page_table, int page_tokens, int64_t n_pages,
                               int64_t n_groups, int group_q, void* out, float* partial, unsigned* counters,
                               unsigned* status, cudaStream_t st, bool pdl, bool allow_cluster, bool counters_zeroed,
                               float* part_out)
{
    if (n_groups <= 0) return cudaSuccess;
    const int G = d.n_q_heads / d.n_kv_heads;
    const int rows = G * group_q;
    if (rows > 32 || n_groups > INT_MAX) return cudaErrorInvalidValue;
    int dev = 0;
    cudaGetDevice(&dev);
    const int nt = nt_for_rows(rows);
    if (!configure(dev, nt)) return cudaErrorInvalidValue;
    const int64_t pairs = n_groups * d.n_kv_heads;
    int bs_log2 = 0;
    while ((1 << bs_log2) < d.block_size) ++bs_log2;
    const Plan p = plan(dev, pairs, rows, allow_cluster, kTT >> bs_log2);
    if (p.n_split > 1 && !p.cluster && !counters_zeroed) {
        // the last split of a pair resets its counter, but a call cannot rely on the
        // previous one having completed every merge
        const cudaError_t e = cudaMemsetAsync(counters, 0, (size_t)pairs * 4, st);
        if (e != cudaSuccess) return e;
    }
    const float scale = d.softmax_scale > 0.f ? d.softmax_scale : 1.0f / sqrtf((float)d.head_dim);
    const float scale_log2 = scale * 1.4426950408889634f;
    const int64_t table_ld = page_table ? d.kv_capacity / page_tokens : 0;

    cudaLaunchConfig_t cfg = {};
    const bool grp_fast = p.n_split == 1;  // queries fastest: one KV head's blocks at a time
    if (!grp_fast && n_groups > 65535) return cudaErrorInvalidValue;
    cfg.gridDim = grp_fast ? dim3((unsigned)n_groups, (unsigned)d.n_kv_heads, 1u)
                           : dim3((unsigned)p.n_split, (unsigned)d.n_kv_heads, (unsigned)n_groups);
    cfg.blockDim = dim3(128 * nwg_for(nt));
    cfg.dynamicSmemBytes = (size_t)p.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    if (p.cluster) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = (unsigned)p.n_split;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.attrs = na ? attr : nullptr;
    cfg.numAttrs = na;
    const int merge = p.n_split == 1 ? 0 : p.cluster ? 1 : 2;
    auto go = [&](auto kern) {
        return cudaLaunchKernelEx(&cfg, kern, (const uint4*)q, (const uint16_t*)k_cache, (const uint16_t*)v_cache,
                                  q_seq, q_pos, sel_idx, sel_cnt, page_table, page_tokens, table_ld, n_pages, d.batch,
                                  d.n_q_heads, d.n_kv_heads, d.kv_capacity, bs_log2, d.top_k, group_q, scale_log2,
                                  p.ips, p.n_split, p.stages, merge, grp_fast ? 1 : 0, (__nv_bfloat16*)out, part_out,
                                  partial, counters,
                                  status);
    };
    return nt == 1 ? go(k_sparse_attn<1, 2>) : nt == 2 ? go(k_sparse_attn<2, 2>) : go(k_sparse_attn<4, 1>);
}

}  // namespace qsa
