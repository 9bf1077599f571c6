// Prefill indexer scoring and top-512 selection on the tcgen05 tensor cores
// (steps 2 and 3 of the QSA layer for chunks of queries: prefill).
//
// blog.cecily.jp/6295 (Raschka's explainer paragraph) and keieiax.jp glossary
// "Qwen Sparse Attention" (section on 4-token micro-blocks): every query scores
// every complete causal block with a light indexer and keeps the best 512.  For a
// chunk of queries this is a dense contraction: per 128-query tile and indexer
// head h, S_h = Q_h (128 x 64) . P^T (64 x N) over the pooled keys P, then
// score = sum_h w_h ReLU(S_h).  The score matrix (8 GiB at 8,192 queries x 1M
// tokens) is never stored: each CTA streams its range of pooled keys and keeps,
// per query row, only the blocks that can still be in the row's top 512.
//
// A 128-query tile may hold rows of several sequences (ragged chunks in one call):
// the CTA then makes one pass over the pooled keys per distinct sequence, and a row
// scores only in its own sequence's pass.
//
// CTA = 10 warps, one CTA per SM (512 TMEM columns):
//   warp 0      TMA producer: the 4 query tiles once, then 128-block pooled tiles
//               (16 KiB, 128-byte swizzle) into a 4-deep ring;
//   warp 1      TMEM allocator and MMA issuer: per pooled tile, 4 heads x 4 K-steps of
//               tcgen05.mma (M=128, N=128, K=16, bf16 -> f32): heads 0 and 1 into
//               accumulator buffer A (TMEM columns 0..255), heads 2 and 3 into buffer
//               B (256..511), so the next tile's first head pair is computed while the
//               epilogue reads this tile's second (N=128 runs the tensor pipe at its
//               full rate, N=64 at two thirds, and halves the MMAs issued per block);
//   warps 2..9  epilogue, two warpgroups: warpgroup g takes columns 64g..64g+63 of
//               every tile; each thread owns one query row (its TMEM lane): tcgen05.ld
//               of buffer A, the partial sum w0 ReLU(s0) + w1 ReLU(s1) (packed f32x2
//               FMAs), buffer A released, then buffer B completes the chain with heads
//               2 and 3 and is released; causal cut, streaming admission.
//
// Two launches per chunk.  A sampling launch scores every 16th block and only
// histograms each row's scores (1/16-octave bins of the order-preserving key).
// The main launch starts each row's admission threshold at the lower edge of the
// bin holding its 64th-best sampled score (about 1,000 blocks of the row expected
// above it; it lies above the row's 512th-best block only when at least 64 samples
// fall among the 512 best blocks, a binomial with mean 32: probability about 4e-7)
// and then raises it as admitted scores fill a histogram: once `need`
// admitted blocks of a thread lie at or above a bin edge, no later block below it
// can reach the top 512, and (blocks arrive in increasing index order) a later
// block equal to it loses every tie, so the thread's own cut is strict.  Thresholds
// are shared, non-strictly, through a global atomic max per row.  The sampled start
// is only an estimate: the finishing select checks that at least 512 blocks cleared
// it and sends the row to the exact fallback otherwise.
//
// All waits are bounded (a global-timer limit); on a timeout the kernel records
// QSA_DEV_TIMEOUT, drains its own copies and MMAs, frees TMEM and returns.

#include <atomic>
#include <cfloat>
#include <mutex>

#include <cudaTypedefs.h>

#include "select_finish.cuh"
#include "sm100_ptx.cuh"

namespace qsa {

using namespace sm100;

namespace {

constexpr int kM = 128;                 // query rows per CTA
constexpr int kN = 128;                 // pooled blocks per tile
constexpr int kNumB = 4;                // pooled-tile ring depth
constexpr int kEpiWarps = 8;
constexpr int kK3Threads = 64 + 32 * kEpiWarps;
constexpr uint32_t kTmemCols = 512;
constexpr int kHistBins = 64;
constexpr int kHistShift = 19;          // main pass: 1/16-octave bins of the orderable key
constexpr int kSampleShift = 19;        // sampling pass: 1/16-octave bins (a 4-octave window)
constexpr int kRaiseEvery = 32;         // admissions between threshold updates
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s bound on any single wait
constexpr int kSampleStride = 16;
constexpr int kSampleKth = 64;
constexpr int kShistWords = kHistBins + 1;   // per (row, CTA, warpgroup): window base, then counts
constexpr uint32_t kNoWindow = 0xFFFFFFFFu;  // window base of a sampler that saw no score

struct __align__(1024) K3Smem {
    __nv_bfloat16 a[kIdxHeads][kM * kIdxDim];   // 4 x 16 KiB
    __nv_bfloat16 b[kNumB][kN * kIdxDim];       // 4 x 16 KiB
    uint32_t hist[2][kHistBins][kM];            // 64 KiB, counter-major per warpgroup
    float w[kM][kIdxHeads];
    int n_c[kM];
    int row_seq[kM];     // sequence of each row, -1 for rows that score nothing
    int pass_seq[kM];    // distinct sequences of the tile, in order of first appearance
    int pass_ncmax[kM];  // longest row of each pass
    int n_pass;
    uint64_t full[kNumB], empty[kNumB];
    uint64_t tmem_full[2], tmem_empty[2];       // accumulator buffers A (heads 0, 1) and B (heads 2, 3)
    uint64_t a_full, mma_done;
    uint32_t tmem_base;
    int error;
};

__device__ __forceinline__ uint64_t now_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait: polls until the phase completes, the CTA's error flag is set, or
// kWaitNs passes (then sets the flag).  Returns true only if the phase completed.
__device__ __forceinline__ bool wait_phase(uint64_t* bar, uint32_t parity, volatile int* error, unsigned* status)
{
    if (mbar_try_wait(bar, parity)) return true;  // fast path: no timer read
    uint64_t t0 = 0;
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 0u) {
            if (*error) return false;
            const uint64_t t = now_ns();
            if (t0 == 0) {
                t0 = t;
            } else if (t - t0 > kWaitNs) {
                *error = 1;
                set_status(status, QSA_DEV_TIMEOUT);
                return false;
            }
        }
    }
}

// v[c] for a run-time c without local memory: a 5-level tree of selects.
__device__ __forceinline__ float pick32(const float (&v)[32], int c)
{
    float a[16], b[8], d[4], e[2];
#pragma unroll
    for (int i = 0; i < 16; ++i) a[i] = (c & 16) ? v[i + 16] : v[i];
#pragma unroll
    for (int i = 0; i < 8; ++i) b[i] = (c & 8) ? a[i + 8] : a[i];
#pragma unroll
    for (int i = 0; i < 4; ++i) d[i] = (c & 4) ? b[i + 4] : b[i];
#pragma unroll
    for (int i = 0; i < 2; ++i) e[i] = (c & 2) ? d[i + 2] : d[i];
    return (c & 1) ? e[1] : e[0];
}

__device__ __forceinline__ float key_to_float(unsigned k)
{
    return __uint_as_float((k & 0x80000000u) ? (k ^ 0x80000000u) : ~k);
}

__device__ __forceinline__ unsigned long long pack2(float lo, float hi)
{
    return ((unsigned long long)__float_as_uint(hi) << 32) | __float_as_uint(lo);
}

__device__ __forceinline__ unsigned long long fma2(unsigned long long a, unsigned long long b, unsigned long long c)
{
    unsigned long long d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

__device__ __forceinline__ float max3(float a, float b, float c)
{
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// 32 consecutive TMEM columns of this thread's lane (two 16-column loads; the caller waits).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32])
{
    float lo[16], hi[16];
    tmem_ld16(taddr, lo);
    tmem_ld16(taddr + 16, hi);
#pragma unroll
    for (int c = 0; c < 16; ++c) {
        v[c] = lo[c];
        v[16 + c] = hi[c];
    }
}

// Two heads of 32 columns of one row folded into the score chain (the same FMA
// order as the decode scorer: w0*r0, then + w1*r1, + w2*r2, + w3*r3), two columns
// per packed f32x2 FMA: acc[c] = wb * ReLU(b[c]) + (wa * ReLU(a[c]) + (cont ? acc[c] : 0)).
__device__ __forceinline__ void pair_scores32(const float (&a)[32], const float (&b)[32], unsigned long long wa,
                                              unsigned long long wb, float (&acc)[32], bool cont)
{
#pragma unroll
    for (int c = 0; c < 32; c += 2) {
        unsigned long long s = cont ? pack2(acc[c], acc[c + 1]) : 0ull;
        s = fma2(wa, pack2(fmaxf(a[c], 0.f), fmaxf(a[c + 1], 0.f)), s);
        s = fma2(wb, pack2(fmaxf(b[c], 0.f), fmaxf(b[c + 1], 0.f)), s);
        acc[c] = __uint_as_float((unsigned)s);
        acc[c + 1] = __uint_as_float((unsigned)(s >> 32));
    }
}

}  // namespace

template <bool kSample>
__global__ void __launch_bounds__(kK3Threads, 1)
k_prefill_scores_tc(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_p,
                    const float* __restrict__ w, const int32_t* __restrict__ q_seq,
                    const int32_t* __restrict__ q_pos, int32_t n_q, int32_t batch, int64_t kv_capacity,
                    int64_t max_blocks, int bs, int top_k, int n_split, int seg_cap, uint32_t* __restrict__ shist,
                    unsigned long long* __restrict__ cand, unsigned* __restrict__ cand_cnt,
                    unsigned* __restrict__ theta_g, unsigned* status)
{
    constexpr int bstride = kSample ? kSampleStride : 1;
    extern __shared__ uint8_t smem_raw[];
    K3Smem& S = *reinterpret_cast<K3Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int split = blockIdx.x, mtile = blockIdx.y;
    const int64_t row0 = (int64_t)mtile * kM;

    // ---- setup: barriers, row metadata, TMEM ----
    if (tid == 0) {
        for (int i = 0; i < kNumB; ++i) {
            mbar_init(&S.full[i], 1);
            mbar_init(&S.empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.tmem_full[i], 1);
            mbar_init(&S.tmem_empty[i], kEpiWarps);  // every epilogue warp reads both buffers
        }
        mbar_init(&S.a_full, 1);
        mbar_init(&S.mma_done, 1);
        S.error = 0;
        fence_mbar_init();
    }
    for (int k = tid; k < 2 * kHistBins * kM; k += kK3Threads) (&S.hist[0][0][0])[k] = 0;
    if (tid < kM) {
        const int64_t r = row0 + tid;
        int nc = 0, seq = -1;
        if (r < n_q) {
            const int s = q_seq[r], t = q_pos[r];
            const bool ok = s >= 0 && s < batch && t >= 0 && (int64_t)t < kv_capacity;
            if (!ok && split == 0 && !kSample) set_status(status, (s < 0 || s >= batch) ? QSA_DEV_BAD_SEQ : QSA_DEV_BAD_POS);
            if (ok) {
                int64_t c = ((int64_t)t + 1) / bs;
                if (c > max_blocks) {
                    if (split == 0 && !kSample) set_status(status, QSA_DEV_BLOCKS_OVER);
                    c = max_blocks;
                }
                nc = (int)c;
                seq = nc > 0 ? s : -1;
            }
#pragma unroll
            for (int h = 0; h < kIdxHeads; ++h) S.w[tid][h] = w[r * kIdxHeads + h];
        }
        S.n_c[tid] = nc;
        S.row_seq[tid] = seq;
    }
    __syncthreads();
    if (tid == 0) {
        // one pass over the pooled keys per distinct sequence of the tile (a chunk of one
        // sequence: a single pass; a tile straddling two chunks: two)
        int np = 0;
        for (int r = 0; r < kM; ++r) {
            const int sq = S.row_seq[r];
            if (sq < 0) continue;
            int p = np - 1;
            if (p < 0 || S.pass_seq[p] != sq) {
                p = 0;
                while (p < np && S.pass_seq[p] != sq) ++p;
                if (p == np) {
                    S.pass_seq[np] = sq;
                    S.pass_ncmax[np] = 0;
                    ++np;
                }
            }
            S.pass_ncmax[p] = max(S.pass_ncmax[p], S.n_c[r]);
        }
        S.n_pass = np;
    }
    if (warp == 1) {
        tmem_alloc(&S.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // per pass, this CTA's range of scored positions (every bstride-th block when
    // sampling): a 1/n_split share of the pass's longest row; stages are numbered
    // across passes (J) for the ring slots and the TMEM stages
    const int n_pass = S.n_pass;
    auto pass_range = [&](int p, int& blk0, int& n_st) {
        const int ncm = (S.pass_ncmax[p] + bstride - 1) / bstride;
        const int chunk = (((ncm + n_split - 1) / n_split) + kN - 1) / kN * kN;
        blk0 = split * chunk;
        const int blk1 = min(blk0 + chunk, ncm);
        n_st = blk1 > blk0 ? (blk1 - blk0 + kN - 1) / kN : 0;
    };
    int n_stages = 0;
    for (int p = 0; p < n_pass; ++p) {
        int b0_, n_st;
        pass_range(p, b0_, n_st);
        n_stages += n_st;
    }
    const uint32_t tmem = S.tmem_base;
    volatile int* err = &S.error;
    const int64_t seq_rows = (kv_capacity / bs) / bstride;  // pooled rows per sequence in the view

    if (warp == 0) {
        if (lane == 0 && n_stages > 0) {
            prefetch_tensormap(&tmap_q);
            prefetch_tensormap(&tmap_p);
            mbar_arrive_expect_tx(&S.a_full, kIdxHeads * kM * kIdxDim * 2);
            for (int h = 0; h < kIdxHeads; ++h) tma_load_3d(S.a[h], &tmap_q, &S.a_full, 0, h, (int)row0);
            int issued = 0;
            for (int p = 0, J = 0; p < n_pass && !*err; ++p) {
                int blk0, n_st;
                pass_range(p, blk0, n_st);
                const int64_t prow0 = (int64_t)S.pass_seq[p] * seq_rows;
                for (int j = 0; j < n_st; ++j, ++J) {
                    const int slot = J % kNumB;
                    if (J >= kNumB && !wait_phase(&S.empty[slot], ((J / kNumB) - 1) & 1, err, status)) break;
                    mbar_arrive_expect_tx(&S.full[slot], kN * kIdxDim * 2);
                    tma_load_2d(S.b[slot], &tmap_p, &S.full[slot], 0, (int)(prow0 + blk0 + (int64_t)j * kN));
                    issued = J + 1;
                }
            }
            if (*err) {
                // drain: every issued tile and the query tiles must land before the CTA exits
                const uint64_t t0 = now_ns();
                while (!mbar_try_wait(&S.a_full, 0) && now_ns() - t0 < kWaitNs) {
                }
                for (int j = max(0, issued - kNumB); j < issued; ++j) {
                    const uint64_t t1 = now_ns();
                    while (!mbar_try_wait(&S.full[j % kNumB], (j / kNumB) & 1) && now_ns() - t1 < kWaitNs) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && n_stages > 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(kM, kN);
            uint64_t adesc[kIdxHeads];
#pragma unroll
            for (int h = 0; h < kIdxHeads; ++h) adesc[h] = smem_desc_sw128(smem_u32(S.a[h]));
            if (wait_phase(&S.a_full, 0, err, status)) {
                for (int j = 0; j < n_stages; ++j) {  // every pass's stages in order
                    const int slot = j % kNumB;
                    if (!wait_phase(&S.full[slot], (j / kNumB) & 1, err, status)) break;
                    const uint64_t bdesc = smem_desc_sw128(smem_u32(S.b[slot]));
                    bool ok = true;
                    for (int pr = 0; pr < 2 && ok; ++pr) {
                        // head pair pr into buffer pr, once the epilogue has read the previous tile's
                        if (j >= 1 && !wait_phase(&S.tmem_empty[pr], (j - 1) & 1, err, status)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        // K-step outer, head inner: consecutive MMAs write different accumulators
#pragma unroll
                        for (int k = 0; k < kIdxDim / 16; ++k)
#pragma unroll
                            for (int hh = 0; hh < 2; ++hh)
                                mma_bf16_ss(tmem + pr * 256 + hh * kN, adesc[2 * pr + hh] + 2 * k, bdesc + 2 * k, idesc,
                                            k > 0);
                        mma_commit(&S.tmem_full[pr]);
                    }
                    if (!ok) break;
                    mma_commit(&S.empty[slot]);
                }
            }
            // every MMA issued must finish before TMEM is released
            mma_commit(&S.mma_done);
            const uint64_t t0 = now_ns();
            while (!mbar_try_wait(&S.mma_done, 0) && now_ns() - t0 < kWaitNs) {
            }
        }
    } else {
        // ---------------- epilogue: warpgroup g takes tiles j with (j & 1) == g ----------------
        const int wg = (warp - 2) >> 2;
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const int64_t row_g = row0 + row;
        const int nc_own = (S.n_c[row] + bstride - 1) / bstride;  // scored positions of this row
        const int my_seq = S.row_seq[row];
        const bool live_any = row_g < n_q && nc_own > 0;
        const float wf0 = S.w[row][0], wf1 = S.w[row][1], wf2 = S.w[row][2], wf3 = S.w[row][3];
        const unsigned long long w0 = pack2(wf0, wf0), w1 = pack2(wf1, wf1), w2 = pack2(wf2, wf2),
                                 w3 = pack2(wf3, wf3);
        uint32_t* hist = &S.hist[wg][0][0] + row;  // counter k at hist[k * kM]
        int wb = -1;                               // histogram window base (absolute bin)
        unsigned wcount = 0;                       // keys counted in the window
        const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16);  // this warp's 32 TMEM lanes

        // ---- main-pass state ----
        unsigned long long* seg = cand + ((row_g * n_split + split) * 2 + wg) * (int64_t)seg_cap;
        unsigned theta_key = 0x00800000u;  // key of -FLT_MAX: every finite score passes
        unsigned cnt = 0, since = 0;
        if (!kSample && shist && live_any && S.n_c[row] > 2 * top_k) {
            // starting threshold: lower edge of the bin holding the row's kSampleKth-best
            // sampled score (merge of the windows of every sampling CTA and warpgroup;
            // a window that saw no sample has base kNoWindow)
            const uint32_t* hw = shist + row_g * 2 * n_split * kShistWords;
            const int nw = 2 * n_split;
            int lo = INT_MAX, hi = -1;
            for (int k = 0; k < nw; ++k) {
                const uint32_t bw = hw[k * kShistWords];
                if (bw == kNoWindow) continue;
                lo = min(lo, (int)bw);
                hi = max(hi, (int)bw + kHistBins - 1);
            }
            unsigned cum = 0;
            for (int bin = hi; bin >= lo && bin >= 0; --bin) {
                for (int k = 0; k < nw; ++k) {
                    const uint32_t bw = hw[k * kShistWords];
                    const int i = bin - (int)bw;
                    if (bw != kNoWindow && i >= 0 && i < kHistBins) cum += hw[k * kShistWords + 1 + i];
                }
                if (cum >= (unsigned)kSampleKth) {
                    const unsigned edge = (unsigned)bin << kSampleShift;
                    if (edge > theta_key) theta_key = edge;
                    break;
                }
            }
        }
        float theta_f = key_to_float(theta_key);

        bool stop = false;
        for (int p = 0, J = 0; p < n_pass && !stop; ++p) {
            int blk0, n_st;
            pass_range(p, blk0, n_st);
            // rows of other sequences score nothing in this pass
            const int nc = my_seq == S.pass_seq[p] ? nc_own : 0;
            const bool live = live_any && nc > 0;
            for (int jp = 0; jp < n_st; ++jp, ++J) {
                const int j = jp;  // stage within the pass
                // buffer A: heads 0 and 1 of this warpgroup's 64 columns -> partial sums
                if (!wait_phase(&S.tmem_full[0], J & 1, err, status)) {
                    stop = true;
                    break;
                }
                tc_fence_after();
                if (!kSample && (J & 7) == 7 && live) {
                    const unsigned g = __ldcg(theta_g + row_g);
                    if (g > theta_key) {
                        theta_key = g;
                        theta_f = key_to_float(theta_key);
                    }
                }
                float part0[32], part1[32];  // columns 0..31 and 32..63 of this warpgroup's share
                {
                    float a0[32], a1[32];
                    tmem_ld32(tbase + 0 * kN + wg * 64, a0);
                    tmem_ld32(tbase + 1 * kN + wg * 64, a1);
                    tmem_ld_wait();
                    pair_scores32(a0, a1, w0, w1, part0, false);
                    tmem_ld32(tbase + 0 * kN + wg * 64 + 32, a0);
                    tmem_ld32(tbase + 1 * kN + wg * 64 + 32, a1);
                    tmem_ld_wait();
                    pair_scores32(a0, a1, w0, w1, part1, false);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.tmem_empty[0]);
                // buffer B: heads 2 and 3 complete the chain w0 r0 + w1 r1 + w2 r2 + w3 r3
                if (!wait_phase(&S.tmem_full[1], J & 1, err, status)) {
                    stop = true;
                    break;
                }
                tc_fence_after();
                {
                    float a2[32], a3[32];
                    tmem_ld32(tbase + 2 * kN + wg * 64, a2);
                    tmem_ld32(tbase + 3 * kN + wg * 64, a3);
                    tmem_ld_wait();
                    pair_scores32(a2, a3, w2, w3, part0, true);
                    tmem_ld32(tbase + 2 * kN + wg * 64 + 32, a2);
                    tmem_ld32(tbase + 3 * kN + wg * 64 + 32, a3);
                    tmem_ld_wait();
                    pair_scores32(a2, a3, w2, w3, part1, true);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.tmem_empty[1]);
                if (!live) continue;
#pragma unroll 1
                for (int half = 0; half < 2; ++half) {
                    float sc[32];
#pragma unroll
                    for (int c = 0; c < 32; ++c) sc[c] = half ? part1[c] : part0[c];
                    const int b_base = blk0 + j * kN + wg * 64 + half * 32;
                    if (b_base + 32 > nc) {
#pragma unroll
                        for (int c = 0; c < 32; ++c)
                            if (b_base + c >= nc) sc[c] = -INFINITY;
                    }
                    if (kSample) {
                        // histogram of every sampled score within 4 octaves of the largest seen
                        float m = sc[0];
#pragma unroll
                        for (int c = 1; c < 31; c += 2) m = max3(m, sc[c], sc[c + 1]);
                        m = fmaxf(m, sc[31]);
                        if (m == -INFINITY) continue;
                        if (wb < 0) wb = max((int)(orderable_key(m) >> kSampleShift) - (kHistBins - 4), 0);
                        const int top = (int)(orderable_key(m) >> kSampleShift);
                        if (top - wb >= kHistBins) {  // slide the window up under the largest score
                            const int d = top - wb - (kHistBins - 4);
                            for (int k = 0; k < kHistBins; ++k) hist[k * kM] = k + d < kHistBins ? hist[(k + d) * kM] : 0u;
                            wb += d;
                        }
#pragma unroll
                        for (int c = 0; c < 32; ++c) {
                            const int jj = (int)(orderable_key(sc[c]) >> kSampleShift) - wb;
                            if (sc[c] != -INFINITY && jj >= 0) hist[jj * kM] += 1;
                        }
                        continue;
                    }
                    float m = sc[0];
#pragma unroll
                    for (int c = 1; c < 31; c += 2) m = max3(m, sc[c], sc[c + 1]);
                    m = fmaxf(m, sc[31]);
                    if (!(m >= theta_f)) continue;
                    unsigned pass = 0;
#pragma unroll
                    for (int c = 0; c < 32; ++c) pass |= (sc[c] >= theta_f ? 1u : 0u) << c;
                    // admissions: columns in increasing block order
                    while (pass) {
                        const int c = __ffs(pass) - 1;
                        pass &= pass - 1;
                        const float sv = pick32(sc, c);
                        if (!(sv >= theta_f)) continue;  // the threshold may have risen within this tile
                        const unsigned key = orderable_key(sv);
                        if (cnt < (unsigned)seg_cap) seg[cnt] = ((unsigned long long)key << 32) | (unsigned)(b_base + c);
                        ++cnt;
                        // the raise histogram only matters once this segment holds many blocks
                        if (cnt < (unsigned)(top_k >> 1)) continue;
                        const int bin = (int)(key >> kHistShift);
                        if (wb < 0) wb = max(bin - 56, 0);
                        int jj = bin - wb;
                        if (jj >= kHistBins) {  // keep the window under the largest score seen
                            const int d = jj - 56;
                            unsigned kept = 0;
                            for (int k = 0; k < kHistBins; ++k) {
                                const unsigned v = k + d < kHistBins ? hist[(k + d) * kM] : 0u;
                                hist[k * kM] = v;
                                kept += v;
                            }
                            wcount = kept;
                            wb += d;
                            jj = 56;
                        }
                        if (jj >= 0) {
                            hist[jj * kM] += 1;
                            ++wcount;
                        }
                        if (++since >= kRaiseEvery && wcount >= (unsigned)top_k + kRaiseEvery) {
                            since = 0;
                            // largest q with (keys counted in bins >= q) >= top_k, scanning up from the bottom
                            unsigned above = wcount;
                            int q = 0;
                            while (q < kHistBins - 1) {
                                const unsigned hq = hist[q * kM];
                                if (above - hq < (unsigned)top_k) break;
                                above -= hq;
                                ++q;
                            }
                            if (q >= 1) {
                                const unsigned edge_key = (unsigned)(wb + q) << kHistShift;
                                if (edge_key + 1 > theta_key) {
                                    theta_key = edge_key + 1;  // strict for this thread's later blocks
                                    theta_f = key_to_float(theta_key);
                                }
                                atomicMax(theta_g + row_g, edge_key);
                                for (int k = 0; k < kHistBins; ++k)
                                    hist[k * kM] = k + q < kHistBins ? hist[(k + q) * kM] : 0u;
                                wcount = above;
                                wb += q;
                            }
                        }
                    }
                }
            }
        }
        if (kSample) {
            if (row_g < n_q) {
                uint32_t* out = shist + ((row_g * n_split + split) * 2 + wg) * kShistWords;
                out[0] = wb < 0 ? kNoWindow : (uint32_t)wb;
                for (int k = 0; k < kHistBins; ++k) out[1 + k] = wb < 0 ? 0u : hist[k * kM];
            }
        } else if (row_g < n_q) {
            cand_cnt[(row_g * n_split + split) * 2 + wg] = cnt;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Gather a row's admitted entries with key >= th from its 2*n_split segments into
// s_cand (up to kCandCap); *n gets the count (may exceed kCandCap), *fail is set if
// a segment overflowed.  Counts are read in parallel, then one flattened pass.
__device__ __forceinline__ void gather_segments(const unsigned long long* __restrict__ cand,
                                                const unsigned* __restrict__ cand_cnt, int64_t r, int n_split,
                                                int seg_cap, unsigned th, unsigned long long* s_cand, int* n,
                                                int* fail)
{
    __shared__ unsigned s_off[2 * 8 + 1];
    const int tid = threadIdx.x;
    const int nseg = 2 * n_split;
    if (tid < nseg) {
        const unsigned c = cand_cnt[r * nseg + tid];
        if (c > (unsigned)seg_cap) *fail = 1;
        s_off[tid + 1] = min(c, (unsigned)seg_cap);
    }
    __syncthreads();
    if (tid == 0) {
        s_off[0] = 0;
        for (int sg = 0; sg < nseg; ++sg) s_off[sg + 1] += s_off[sg];
    }
    __syncthreads();
    const unsigned total = s_off[nseg];
    const int64_t base = r * nseg * (int64_t)seg_cap;
    const int lane = tid & 31;
    // one shared-memory atomic per warp and round (ballot + prefix), not one per entry
    for (unsigned k0 = 0; k0 < total; k0 += 256) {
        const unsigned k = k0 + tid;
        unsigned long long e = 0ull;
        if (k < total) {
            int sg = 0;
            while (sg + 1 < nseg && s_off[sg + 1] <= k) ++sg;
            e = __ldg(cand + base + (int64_t)sg * seg_cap + (k - s_off[sg]));
        }
        const bool take = k < total && (unsigned)(e >> 32) >= th;
        const unsigned m = __ballot_sync(0xffffffffu, take);
        if (!m) continue;
        const int leader = __ffs(m) - 1;
        int slot0 = 0;
        if (lane == leader) slot0 = atomicAdd(n, __popc(m));
        slot0 = __shfl_sync(0xffffffffu, slot0, leader);
        if (take) {
            const int slot = slot0 + __popc(m & ((1u << lane) - 1u));
            if (slot < kCandCap) s_cand[slot] = e;
        }
    }
    __syncthreads();
}


// ---------------------------------------------------------------- finishing select

// One CTA per query row: exact top 512 among the row's admitted blocks (keys at
// or above the row's final threshold), or every block when n_c <= 512.  Rows whose
// segments overflowed, or whose survivors do not fit the shared-memory finisher,
// go to the worklist of k_prefill_fallback.
__global__ void __launch_bounds__(256, 3)  // three rows per SM
k_prefill_finish(const int32_t* __restrict__ q_seq, const int32_t* __restrict__ q_pos, int32_t n_q, int32_t batch,
                 int64_t kv_capacity, int64_t max_blocks, int bs, int top_k, int n_split, int seg_cap,
                 const unsigned long long* __restrict__ cand, const unsigned* __restrict__ cand_cnt,
                 const unsigned* __restrict__ theta_g, int32_t* __restrict__ worklist, int32_t* __restrict__ sel_idx,
                 int32_t* __restrict__ sel_cnt)
{
    __shared__ FinishSmem S;
    extern __shared__ unsigned long long s_cand[];  // kCandCap entries (dynamic)
    __shared__ int s_n, s_fail;
    const int tid = threadIdx.x;
    const int64_t r = blockIdx.x;
    const int s = q_seq[r], t = q_pos[r];
    const bool ok = s >= 0 && s < batch && t >= 0 && (int64_t)t < kv_capacity;
    const int64_t n_c = ok ? min(((int64_t)t + 1) / bs, max_blocks) : 0;
    int32_t* out = sel_idx + r * kSelCap;
    if (n_c <= top_k) {
        for (int k = tid; k < kSelCap; k += 256) out[k] = k < n_c ? k : -1;
        if (tid == 0) sel_cnt[r] = (int)n_c;
        return;
    }
    const unsigned theta = theta_g[r];
    if (tid == 0) {
        s_n = 0;
        s_fail = 0;
    }
    for (int k = tid; k < kSelCap; k += 256) S.list[k] = INT_MAX;
    if (tid == 0) S.n_list = 0;
    __syncthreads();
    gather_segments(cand, cand_cnt, r, n_split, seg_cap, theta, s_cand, &s_n, &s_fail);
    const int nc = s_n;
    if (s_fail || nc > kCandCap || nc < top_k) {
        if (tid == 0) worklist[1 + atomicAdd(worklist, 1)] = (int32_t)r;
        return;
    }
    unsigned long long cr[kPerThreadCand];
#pragma unroll
    for (int k = 0; k < kPerThreadCand; ++k) {
        const int j = tid + 256 * k;
        cr[k] = j < nc ? s_cand[j] : 0ull;
    }
    const Cut cut = resolve_cut_regs(S, cr, nc, top_k, true, 0u);
    if (!take_by_cut(S, cr, nc, cut)) {
        if (tid == 0) worklist[1 + atomicAdd(worklist, 1)] = (int32_t)r;
        return;
    }
    sort_list_512(S);
    for (int k = tid; k < kSelCap; k += 256) out[k] = k < top_k ? S.list[k] : -1;
    if (tid == 0) sel_cnt[r] = top_k;
}

// Rows the streaming pass could not settle: recompute the row's scores with CUDA
// cores into scratch, then select in block order.  Persistent over the worklist.
__global__ void __launch_bounds__(256)
k_prefill_fallback(const __nv_bfloat16* __restrict__ q_idx, const float* __restrict__ w,
                   const __nv_bfloat16* __restrict__ pooled, const int32_t* __restrict__ q_seq,
                   const int32_t* __restrict__ q_pos, int64_t kv_capacity, int64_t max_blocks, int bs, int top_k,
                   const int32_t* __restrict__ worklist, float* __restrict__ scratch, int32_t* __restrict__ sel_idx,
                   int32_t* __restrict__ sel_cnt)
{
    __shared__ FinishSmem S;
    __shared__ float s_q[kIdxHeads][kIdxDim];
    const int tid = threadIdx.x;
    const int n_work = worklist[0];
    float* row_scores = scratch + (int64_t)blockIdx.x * max_blocks;
    for (int wi = blockIdx.x; wi < n_work; wi += gridDim.x) {
        const int64_t r = worklist[1 + wi];
        const int s = q_seq[r], t = q_pos[r];
        const int64_t n_c = min(((int64_t)t + 1) / bs, max_blocks);
        __syncthreads();
        for (int k = tid; k < kIdxHeads * kIdxDim; k += 256)
            s_q[k / kIdxDim][k % kIdxDim] = __bfloat162float(q_idx[r * kIdxHeads * kIdxDim + k]);
        __syncthreads();
        float wv[kIdxHeads];
#pragma unroll
        for (int h = 0; h < kIdxHeads; ++h) wv[h] = w[r * kIdxHeads + h];
        const __nv_bfloat16* prow = pooled + (int64_t)s * (kv_capacity / bs) * kIdxDim;
        for (int64_t b = tid; b < n_c; b += 256) {
            float acc[kIdxHeads] = {0.f, 0.f, 0.f, 0.f};
            const uint4* pk = reinterpret_cast<const uint4*>(prow + b * kIdxDim);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 v = __ldg(pk + c);
                const uint32_t x[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float p0 = bf16lo(x[e]), p1 = bf16hi(x[e]);
#pragma unroll
                    for (int h = 0; h < kIdxHeads; ++h)
                        acc[h] = fmaf(s_q[h][8 * c + 2 * e + 1], p1, fmaf(s_q[h][8 * c + 2 * e], p0, acc[h]));
                }
            }
            float sc = 0.f;
#pragma unroll
            for (int h = 0; h < kIdxHeads; ++h) sc = fmaf(wv[h], fmaxf(acc[h], 0.f), sc);
            row_scores[b] = sc;
        }
        __threadfence_block();
        __syncthreads();
        for (int k = tid; k < kSelCap; k += 256) S.list[k] = INT_MAX;
        __syncthreads();
        select_by_rescan(S, row_scores, n_c, true, 0u, top_k);
        int32_t* out = sel_idx + r * kSelCap;
        const int cnt = (int)min((int64_t)top_k, n_c);
        for (int k = tid; k < kSelCap; k += 256) out[k] = k < cnt ? S.list[k] : -1;
        if (tid == 0) sel_cnt[r] = cnt;
    }
}

// ---------------------------------------------------------------- host side

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

bool set_smem_once(const void* fn, int bytes, std::atomic<bool> (&done)[128])
{
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 128) return false;
    if (!done[dev].load()) {  // setting it twice (two host threads) is harmless
        if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
        done[dev].store(true);
    }
    return true;
}

}  // namespace

int prefill_splits(int32_t n_q, int64_t max_blocks)
{
    const int n_tiles = (n_q + kM - 1) / kM;
    int s = 148 / (n_tiles > 0 ? n_tiles : 1);
    const int64_t stages = (max_blocks + kN - 1) / kN;
    const int64_t cap = stages / 4 > 0 ? stages / 4 : 1;  // at least ~4 tiles of work per CTA
    if (s > cap) s = (int)cap;
    if (s > 8) s = 8;
    return s < 1 ? 1 : s;
}

int prefill_seg_cap() { return 2048; }
int prefill_segments(int n_split) { return 2 * n_split; }
int prefill_shist_words(int n_split) { return 2 * n_split * kShistWords; }

size_t prefill_smem_bytes() { return sizeof(K3Smem) + 1024; }

bool prefill_sampled(const qsa_dims& d, int64_t max_blocks)
{
    return d.kv_capacity % ((int64_t)d.block_size * kSampleStride) == 0 && max_blocks > 2 * d.top_k;
}

cudaError_t launch_prefill_select(const qsa_dims& d, const void* q_idx, const float* w, const void* pooled,
                                  const int32_t* q_seq, const int32_t* q_pos, int32_t n_q, int64_t max_blocks,
                                  int n_split, unsigned long long* cand, unsigned* cand_cnt, unsigned* theta_g,
                                  uint32_t* shist, int32_t* worklist, float* scratch, int n_fallback_ctas,
                                  int32_t* sel_idx, int32_t* sel_cnt, unsigned* status, cudaStream_t st)
{
    if (n_q <= 0) return cudaSuccess;
    auto encode = encode_fn();
    if (!encode) return cudaErrorNotSupported;
    CUtensorMap tq, tp, ts;
    {
        // indexer queries: [n_q][4][64] bf16 as a 3-D tensor (dim, head, query); box = 64 x 1 x 128
        const cuuint64_t dims[3] = {(cuuint64_t)kIdxDim, (cuuint64_t)kIdxHeads, (cuuint64_t)n_q};
        const cuuint64_t strides[2] = {(cuuint64_t)kIdxDim * 2, (cuuint64_t)kIdxHeads * kIdxDim * 2};
        const cuuint32_t box[3] = {(cuuint32_t)kIdxDim, 1u, (cuuint32_t)kM};
        const cuuint32_t estr[3] = {1u, 1u, 1u};
        if (encode(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q_idx), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    const bool sampled = prefill_sampled(d, max_blocks);
    for (int pass = 0; pass < (sampled ? 2 : 1); ++pass) {
        // pooled keys of all sequences: [B * T/4][64] bf16, box = 64 x 64 blocks; the sampling
        // view takes every kSampleStride-th block (row pitch kSampleStride x 128 B)
        const int stride = pass == 0 ? 1 : kSampleStride;
        const cuuint64_t dims[2] = {(cuuint64_t)kIdxDim, (cuuint64_t)(d.batch * (d.kv_capacity / d.block_size) / stride)};
        const cuuint64_t strides[1] = {(cuuint64_t)kIdxDim * 2 * stride};
        const cuuint32_t box[2] = {(cuuint32_t)kIdxDim, (cuuint32_t)kN};
        const cuuint32_t estr[2] = {1u, 1u};
        if (encode(pass == 0 ? &tp : &ts, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(pooled), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    static std::atomic<bool> attr_main[128], attr_sample[128], attr_fin[128];
    const int smem = (int)prefill_smem_bytes();
    if (!set_smem_once((const void*)k_prefill_scores_tc<false>, smem, attr_main) ||
        !set_smem_once((const void*)k_prefill_scores_tc<true>, smem, attr_sample) ||
        !set_smem_once((const void*)k_prefill_finish, (int)(kCandCap * sizeof(unsigned long long)), attr_fin))
        return cudaErrorInvalidValue;
    const int seg_cap = prefill_seg_cap();
    const int n_tiles = (n_q + kM - 1) / kM;
    if (sampled)  // the main pass's CTA grid: each thread histograms its share of its row's samples
        k_prefill_scores_tc<true><<<dim3((unsigned)n_split, (unsigned)n_tiles), kK3Threads, smem, st>>>(
            tq, ts, w, q_seq, q_pos, n_q, d.batch, d.kv_capacity, max_blocks, d.block_size, d.top_k, n_split, 0,
            shist, nullptr, nullptr, nullptr, status);
    k_prefill_scores_tc<false><<<dim3((unsigned)n_split, (unsigned)n_tiles), kK3Threads, smem, st>>>(
        tq, tp, w, q_seq, q_pos, n_q, d.batch, d.kv_capacity, max_blocks, d.block_size, d.top_k, n_split, seg_cap,
        sampled ? shist : nullptr, cand, cand_cnt, theta_g, status);
    k_prefill_finish<<<(unsigned)n_q, 256, kCandCap * sizeof(unsigned long long), st>>>(
        q_seq, q_pos, n_q, d.batch, d.kv_capacity, max_blocks, d.block_size, d.top_k, n_split, seg_cap, cand,
        cand_cnt, theta_g, worklist, sel_idx, sel_cnt);
    k_prefill_fallback<<<(unsigned)n_fallback_ctas, 256, 0, st>>>(
        (const __nv_bfloat16*)q_idx, w, (const __nv_bfloat16*)pooled, q_seq, q_pos, d.kv_capacity, max_blocks,
        d.block_size, d.top_k, worklist, scratch, sel_idx, sel_cnt);
    return cudaGetLastError();
}

}  // namespace qsa
