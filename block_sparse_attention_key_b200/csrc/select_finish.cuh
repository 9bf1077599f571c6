// Block-level (256 threads) exact top-k finishers shared by the decode select
// and the prefill select.  Keys are 32-bit order-preserving encodings of fp32
// scores; the top `need` are taken by (key descending, block index ascending).
// Radix digits: bits 31..20 (4096 bins), 19..8 (4096 bins), 7..0 (256 bins).
#pragma once

#include <climits>

#include "select_common.cuh"

namespace qsa {

constexpr int kPerThreadCand = kCandCap / 256;  // candidates each finishing thread holds
constexpr int kMaxTieRank = 1024;               // keys equal at the cut ranked pairwise at most

// 16-byte aligned: hist doubles as scratch for 64-bit sort keys.
struct alignas(16) FinishSmem {
    unsigned hist[kBins2];
    int list[kSelCap];
    unsigned warp[8];
    int cnt[8];
    int n_list;
    unsigned res_digit, res_count;
    int res_need;
    int neq;
};

// Among candidates counted in S.hist[0 .. 256*kPer) find the digit holding the
// need-th largest: S.res_digit, S.res_need (still wanted inside it), S.res_count.
template <int kPer>
__device__ __forceinline__ void resolve_smem(FinishSmem& S, int need)
{
    const int tid = threadIdx.x;
    unsigned h[kPer];
    unsigned local = 0;
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
        h[k] = S.hist[tid * kPer + k];
        local += h[k];
    }
    const unsigned suf = block_suffix_sum_256(local, S.warp);
    const unsigned after = suf - local;
    if (suf >= (unsigned)need && after < (unsigned)need) {
        unsigned run = after;
        int found = -1;
        unsigned fh = 0, frun = 0;
#pragma unroll
        for (int k = kPer - 1; k >= 0; --k) {
            if (found < 0 && run + h[k] >= (unsigned)need) {
                found = k;
                fh = h[k];
                frun = run;
            }
            run += h[k];
        }
        S.res_digit = (unsigned)(tid * kPer + found);
        S.res_count = fh;
        S.res_need = need - (int)frun;
    }
    __syncthreads();
}

__device__ __forceinline__ void clear_hist(FinishSmem& S, int nbins)
{
    for (int k = threadIdx.x; k < nbins; k += 256) S.hist[k] = 0;
    __syncthreads();
}

// Exclusive prefix sum over the 256 threads of the CTA, in thread order;
// *total gets the sum.  Two barriers.
__device__ __forceinline__ unsigned block_excl_scan_256(unsigned v, unsigned* s_warp /*[8]*/, unsigned* total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const unsigned o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    unsigned before = 0, all = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        const unsigned x = s_warp[w];
        before += w < warp ? x : 0u;
        all += x;
    }
    __syncthreads();
    *total = all;
    return before + incl - v;
}

// Ascending sort of 512 elements a[0..512) by the 256 threads of the CTA, with
// b[0..512) as scratch; the result is left in a.  Each warp first ranks its 64
// elements among themselves (register shuffles, no barrier), then three rounds
// merge sorted runs pairwise (64 -> 128 -> 256 -> 512): an element's place in the
// merged run is its place in its own run plus the number of elements of the
// partner run before it (binary search; a left-run element counts the partner's
// smaller elements, a right-run element also the equal ones, so equal elements
// keep distinct places).
template <typename T>
__device__ __forceinline__ void block_sort_512(T* a, T* b)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    {
        const T e0 = a[64 * warp + lane], e1 = a[64 * warp + 32 + lane];
        int r0 = 0, r1 = 0;
#pragma unroll 8
        for (int j = 0; j < 32; ++j) {
            const T v0 = __shfl_sync(0xffffffffu, e0, j), v1 = __shfl_sync(0xffffffffu, e1, j);
            r0 += (v0 < e0 || (v0 == e0 && j < lane)) ? 1 : 0;
            r0 += v1 < e0 ? 1 : 0;
            r1 += v0 <= e1 ? 1 : 0;
            r1 += (v1 < e1 || (v1 == e1 && j < lane)) ? 1 : 0;
        }
        b[64 * warp + r0] = e0;
        b[64 * warp + r1] = e1;
    }
    __syncthreads();
    T* src = b;
    T* dst = a;
#pragma unroll 1
    for (int L = 64; L < kSelCap; L <<= 1) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int p = tid + 256 * h;
            const T x = src[p];
            const int run = p / L, pos = p % L;
            const bool right = run & 1;
            const T* other = src + (run ^ 1) * L;
            int lo = 0, hi = L;
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                const T v = other[mid];
                if (right ? v <= x : v < x) lo = mid + 1;
                else hi = mid;
            }
            dst[(run & ~1) * L + pos + lo] = x;
        }
        __syncthreads();
        T* t = src;
        src = dst;
        dst = t;
    }
}

// Ascending sort of S.list[0..512) (unused slots hold INT_MAX).
__device__ __forceinline__ void sort_list_512(FinishSmem& S)
{
    block_sort_512<int>(S.list, reinterpret_cast<int*>(S.hist));
}

// Take the top `need` of nc <= 512 candidates (entry = key << 32 | block; key
// descending, then block ascending) by sorting them, and append their blocks to
// S.list after its S.n_list entries.
__device__ __forceinline__ void take_top_sorted(FinishSmem& S, const unsigned long long (&cr)[kPerThreadCand], int nc,
                                                int need)
{
    const int tid = threadIdx.x;
    unsigned long long* a = reinterpret_cast<unsigned long long*>(S.hist);
    unsigned long long* b = a + kSelCap;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int j = tid + 256 * k;
        // ascending order of (~key, block) = key descending, block ascending
        a[j] = j < nc ? ((unsigned long long)(~(unsigned)(cr[k] >> 32)) << 32) | (unsigned)cr[k] : ~0ull;
    }
    __syncthreads();
    block_sort_512<unsigned long long>(a, b);
    const int base = S.n_list;
    for (int j = tid; j < need && base + j < kSelCap; j += 256) S.list[base + j] = (int)(unsigned)a[j];
    __syncthreads();
    if (tid == 0) S.n_list = min(base + need, kSelCap);
    __syncthreads();
}

// The cut of a selection: keys > cut are taken; keys == cut are all taken when
// `whole`, else only the `need` with the lowest block indices.
struct Cut {
    unsigned key;
    int need;
    bool whole;
};

// Resolve the cut among candidates held in registers (kPerThreadCand per thread,
// entry = key << 32 | block, `nc` valid in total).  If `from_digit1` is false all
// candidates share the top 12 bits `p12`.  `need` >= 1 candidates are wanted.
__device__ __forceinline__ Cut resolve_cut_regs(FinishSmem& S, const unsigned long long (&cr)[kPerThreadCand],
                                                int nc, int need, bool from_digit1, unsigned p12)
{
    const int tid = threadIdx.x;
    if (from_digit1) {
        clear_hist(S, kBins1);
#pragma unroll
        for (int k = 0; k < kPerThreadCand; ++k)
            if (tid + 256 * k < nc) atomicAdd(&S.hist[(unsigned)(cr[k] >> 52)], 1u);
        __syncthreads();
        resolve_smem<kBins1 / 256>(S, need);
        p12 = S.res_digit;
        need = S.res_need;
        if (S.res_count == (unsigned)need) {
            __syncthreads();
            return Cut{p12 << 20, need, true};
        }
        __syncthreads();
    }
    clear_hist(S, kBins2);
#pragma unroll
    for (int k = 0; k < kPerThreadCand; ++k)
        if (tid + 256 * k < nc && (unsigned)(cr[k] >> 52) == p12) atomicAdd(&S.hist[(unsigned)(cr[k] >> 40) & 0xFFFu], 1u);
    __syncthreads();
    resolve_smem<kBins2 / 256>(S, need);
    const unsigned p24 = (p12 << 12) | S.res_digit;
    need = S.res_need;
    if (S.res_count == (unsigned)need) {
        __syncthreads();
        return Cut{p24 << 8, need, true};
    }
    __syncthreads();
    clear_hist(S, kBins3);
#pragma unroll
    for (int k = 0; k < kPerThreadCand; ++k)
        if (tid + 256 * k < nc && (unsigned)(cr[k] >> 40) == p24) atomicAdd(&S.hist[(unsigned)(cr[k] >> 32) & 0xFFu], 1u);
    __syncthreads();
    resolve_smem<1>(S, need);
    const Cut c{(p24 << 8) | S.res_digit, S.res_need, S.res_count == (unsigned)S.res_need};
    S.neq = (int)S.res_count;
    __syncthreads();
    return c;
}

// Append the candidates taken by `c` to S.list (after S.n_list existing entries).
// Returns false when too many keys tie at the cut to rank them pairwise.
__device__ __forceinline__ bool take_by_cut(FinishSmem& S, const unsigned long long (&cr)[kPerThreadCand], int nc,
                                            const Cut& c)
{
    const int tid = threadIdx.x;
    if (!c.whole && S.neq > kMaxTieRank) return false;
    int* eq_idx = reinterpret_cast<int*>(S.hist);  // block indices of keys equal to the cut
    __shared__ int s_neq;
    if (tid == 0) s_neq = 0;
    __syncthreads();
    if (!c.whole) {
#pragma unroll
        for (int k = 0; k < kPerThreadCand; ++k)
            if (tid + 256 * k < nc && (unsigned)(cr[k] >> 32) == c.key) eq_idx[atomicAdd(&s_neq, 1)] = (int)(unsigned)cr[k];
    }
    __syncthreads();
    const int neq = s_neq;
    unsigned take_mask = 0;
#pragma unroll
    for (int k = 0; k < kPerThreadCand; ++k) {
        if (tid + 256 * k >= nc) continue;
        const unsigned key = (unsigned)(cr[k] >> 32);
        const int b = (int)(unsigned)cr[k];
        bool take = key > c.key || (key == c.key && c.whole);
        if (!take && key == c.key) {
            int rank = 0;
            for (int j = 0; j < neq; ++j) rank += eq_idx[j] < b;
            take = rank < c.need;
        }
        take_mask |= (take ? 1u : 0u) << k;
    }
    // places in S.list by a block-wide scan of the per-thread counts (no shared atomics)
    unsigned total;
    int slot = S.n_list + (int)block_excl_scan_256((unsigned)__popc(take_mask), S.warp, &total);
#pragma unroll
    for (int k = 0; k < kPerThreadCand; ++k)
        if (take_mask >> k & 1u) {
            if (slot < kSelCap) S.list[slot] = (int)(unsigned)cr[k];
            ++slot;
        }
    __syncthreads();
    if (tid == 0) S.n_list += (int)total;
    __syncthreads();
    return true;
}

// take_by_cut for any number of keys tied at the cut: when too many tie to rank them
// pairwise, the tied candidates' blocks (distinct) are cut by the same radix select
// on ~block, so the `need` lowest blocks are taken.
__device__ inline void take_by_cut_exact(FinishSmem& S, const unsigned long long (&cr)[kPerThreadCand], int nc,
                                         const Cut& c)
{
    if (take_by_cut(S, cr, nc, c)) return;
    const int tid = threadIdx.x;
    unsigned long long tied[kPerThreadCand];
#pragma unroll
    for (int k = 0; k < kPerThreadCand; ++k)
        tied[k] = (tid + 256 * k < nc && (unsigned)(cr[k] >> 32) == c.key)
                      ? (unsigned long long)(~(uint32_t)cr[k]) << 32
                      : 0ull;
    const Cut cb = resolve_cut_regs(S, tied, nc, c.need, true, 0u);  // ~block values are distinct: cb.whole
    unsigned take_mask = 0;
#pragma unroll
    for (int k = 0; k < kPerThreadCand; ++k) {
        if (tid + 256 * k >= nc) continue;
        const unsigned key = (unsigned)(cr[k] >> 32);
        const bool take = key > c.key || (key == c.key && ~(uint32_t)cr[k] >= cb.key);
        take_mask |= (take ? 1u : 0u) << k;
    }
    unsigned total;
    int slot = S.n_list + (int)block_excl_scan_256((unsigned)__popc(take_mask), S.warp, &total);
#pragma unroll
    for (int k = 0; k < kPerThreadCand; ++k)
        if (take_mask >> k & 1u) {
            if (slot < kSelCap) S.list[slot] = (int)(unsigned)cr[k];
            ++slot;
        }
    __syncthreads();
    if (tid == 0) S.n_list += (int)total;
    __syncthreads();
}

// Ordered selection of the top `need` keys of a score row in global memory
// (keys whose top 12 bits exceed `p12` are all taken; among those equal to it the
// top `need12`), written to S.list in ascending block order.  With `from_digit1`
// the whole row is ranked for its top `need12` (p12 is ignored).
__device__ inline void select_by_rescan(FinishSmem& S, const float* srow, int64_t n_c, bool from_digit1, unsigned p12,
                                 int need12)
{
    const int tid = threadIdx.x;
    int need = need12;
    unsigned cut;
    bool whole = false;
    if (from_digit1) {
        clear_hist(S, kBins1);
        for (int64_t b = tid; b < n_c; b += 256) atomicAdd(&S.hist[orderable_key(__ldcg(srow + b)) >> 20], 1u);
        __syncthreads();
        resolve_smem<kBins1 / 256>(S, need);
        p12 = S.res_digit;
        need = S.res_need;
        whole = S.res_count == (unsigned)need;
        __syncthreads();
    }
    cut = p12 << 20;
    if (!whole) {
        clear_hist(S, kBins2);
        for (int64_t b = tid; b < n_c; b += 256) {
            const unsigned key = orderable_key(__ldcg(srow + b));
            if ((key >> 20) == p12) atomicAdd(&S.hist[(key >> 8) & 0xFFFu], 1u);
        }
        __syncthreads();
        resolve_smem<kBins2 / 256>(S, need);
        const unsigned p24 = (p12 << 12) | S.res_digit;
        need = S.res_need;
        cut = p24 << 8;
        whole = S.res_count == (unsigned)need;
        __syncthreads();
        if (!whole) {
            clear_hist(S, kBins3);
            for (int64_t b = tid; b < n_c; b += 256) {
                const unsigned key = orderable_key(__ldcg(srow + b));
                if ((key >> 8) == p24) atomicAdd(&S.hist[key & 0xFFu], 1u);
            }
            __syncthreads();
            resolve_smem<1>(S, need);
            cut = (p24 << 8) | S.res_digit;
            need = S.res_need;
            whole = S.res_count == (unsigned)need;
            __syncthreads();
        }
    }
    int taken = 0, eq_seen = 0;
    for (int64_t base = 0; base < n_c; base += 256) {
        const int64_t b = base + tid;
        const bool valid = b < n_c;
        const unsigned key = valid ? orderable_key(__ldcg(srow + b)) : 0u;
        int eq_total;
        const bool eq = valid && key == cut;
        const int eq_rank = block_rank_256(eq, S.cnt, &eq_total);
        const bool take = valid && (key > cut || (eq && (whole || eq_seen + eq_rank < need)));
        int n_take;
        const int rank = block_rank_256(take, S.cnt, &n_take);
        if (take && taken + rank < kSelCap) S.list[taken + rank] = (int)b;
        taken += n_take;
        eq_seen += eq_total;
    }
    __syncthreads();
    if (tid == 0) S.n_list = taken < kSelCap ? taken : kSelCap;
    __syncthreads();
}


// ---------------------------------------------------------------------------
// Whole-row select by one CTA for rows of at most kRowSmemBlocks scores.  The
// row's keys sit in shared memory, thread t owning blocks [64t, 64t + 64) as 16
// aligned 16-byte words (4 pad words after every 64 keys keep a warp's 16-byte
// reads conflict-free); the 12-12-8 bit radix cut is resolved there and the
// winners are emitted in ascending block order by two block-wide scans (equal
// keys at the cut: lowest block indices first), so nothing is sorted.  The
// digit-1 histogram of the row is complete in `hist1`.
constexpr int kRowSmemBlocks = 16384;
constexpr int kRowSmemWords = kRowSmemBlocks + kRowSmemBlocks / 16;

__device__ __forceinline__ int row_pos(int b) { return b + 4 * (b >> 6); }

__device__ inline void select_row_in_smem(FinishSmem& S, unsigned* keys, const float* srow, int n_c, int top_k,
                                          const unsigned* hist1, int32_t* out, int32_t* cnt_out)
{
    const int tid = threadIdx.x;
    if (n_c <= top_k) {
        for (int k = tid; k < kSelCap; k += 256) out[k] = k < n_c ? k : -1;
        if (tid == 0) *cnt_out = n_c;
        return;
    }
    {
        // keys of the row (written by other CTAs of this grid: read through L2),
        // all loads in flight at once; blocks >= n_c get key 0, below every score
        float4 v[kRowSmemBlocks / 1024];
#pragma unroll
        for (int k = 0; k < kRowSmemBlocks / 1024; ++k) {
            const int b = 4 * tid + 1024 * k;
            v[k] = b < n_c ? __ldcg(reinterpret_cast<const float4*>(srow + b)) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        unsigned h[kBins1 / 256];
#pragma unroll
        for (int k = 0; k < kBins1 / 256; ++k) h[k] = __ldcg(hist1 + tid + 256 * k);
#pragma unroll
        for (int k = 0; k < kRowSmemBlocks / 1024; ++k) {
            const int b = 4 * tid + 1024 * k;
            uint4 kk;
            kk.x = b + 0 < n_c ? orderable_key(v[k].x) : 0u;
            kk.y = b + 1 < n_c ? orderable_key(v[k].y) : 0u;
            kk.z = b + 2 < n_c ? orderable_key(v[k].z) : 0u;
            kk.w = b + 3 < n_c ? orderable_key(v[k].w) : 0u;
            *reinterpret_cast<uint4*>(keys + row_pos(b)) = kk;
        }
#pragma unroll
        for (int k = 0; k < kBins1 / 256; ++k) S.hist[tid + 256 * k] = h[k];
    }
    __syncthreads();
    const uint4* mine = reinterpret_cast<const uint4*>(keys + row_pos(64 * tid));
    // digit 1 (bits 31..20)
    resolve_smem<kBins1 / 256>(S, top_k);
    unsigned cut = S.res_digit << 20;
    int need = S.res_need;
    bool whole = S.res_count == (unsigned)need;
    __syncthreads();
    if (!whole) {
        // digit 2 (bits 19..8) among keys of the boundary bin
        const unsigned p12 = cut >> 20;
        clear_hist(S, kBins2);
#pragma unroll 4
        for (int q = 0; q < 16; ++q) {
            const uint4 k4 = mine[q];
            const unsigned kv[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if ((kv[e] >> 20) == p12) atomicAdd(&S.hist[(kv[e] >> 8) & 0xFFFu], 1u);
        }
        __syncthreads();
        resolve_smem<kBins2 / 256>(S, need);
        const unsigned p24 = (p12 << 12) | S.res_digit;
        cut = p24 << 8;
        need = S.res_need;
        whole = S.res_count == (unsigned)need;
        __syncthreads();
        if (!whole) {
            // digit 3 (bits 7..0)
            clear_hist(S, kBins3);
#pragma unroll 4
            for (int q = 0; q < 16; ++q) {
                const uint4 k4 = mine[q];
                const unsigned kv[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if ((kv[e] >> 8) == p24) atomicAdd(&S.hist[kv[e] & 0xFFu], 1u);
            }
            __syncthreads();
            resolve_smem<1>(S, need);
            cut = (p24 << 8) | S.res_digit;
            need = S.res_need;
            whole = S.res_count == (unsigned)need;
            __syncthreads();
        }
    }
    // keys > cut are taken; keys == cut: all when whole, else the first `need` by index
    unsigned gt = 0, eq = 0;
#pragma unroll 4
    for (int q = 0; q < 16; ++q) {
        const uint4 k4 = mine[q];
        gt += (k4.x > cut) + (k4.y > cut) + (k4.z > cut) + (k4.w > cut);
        eq += (k4.x == cut) + (k4.y == cut) + (k4.z == cut) + (k4.w == cut);
    }
    unsigned eq_total;
    const unsigned eq_before = block_excl_scan_256(eq, S.warp, &eq_total);
    const int take_eq = whole ? (int)eq : max(0, min((int)eq, need - (int)eq_before));
    unsigned n_taken;
    int slot = (int)block_excl_scan_256(gt + (unsigned)take_eq, S.warp, &n_taken);
    int eq_left = take_eq;
    for (int q = 0; q < 16; ++q) {
        const uint4 k4 = mine[q];
        const unsigned kv[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const bool is_eq = kv[e] == cut && eq_left > 0;
            if (kv[e] > cut || is_eq) {
                if (slot < kSelCap) out[slot] = 64 * tid + 4 * q + e;
                ++slot;
            }
            eq_left -= is_eq ? 1 : 0;
        }
    }
    for (int k = (int)n_taken + tid; k < kSelCap; k += 256) out[k] = -1;
    if (tid == 0) *cnt_out = (int)min(n_taken, (unsigned)top_k);
}

}  // namespace qsa
