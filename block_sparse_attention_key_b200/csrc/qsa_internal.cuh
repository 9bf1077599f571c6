// Internal declarations shared by the kernels and the host entry points of
// libqsa.so (B200, sm_100a).  Nothing here is part of the public ABI.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/qsa.h"

namespace qsa {

// ---- fixed method parameters (validated on the host) ----
// micro-block size (dims.block_size) and blocks kept per query (dims.top_k) are
// run-time values: block_size in {1, 2, 4, 8, 16}, 1 <= top_k <= kSelCap
constexpr int kSelCap = 512;     // capacity of a query's selection (and row stride of sel_idx)
constexpr int kMaxBlockSize = 16;
constexpr int kIdxHeads = 4;     // indexer heads
constexpr int kIdxDim = 64;      // indexer head dim
constexpr int kHeadDim = 128;    // main attention head dim
constexpr int kMaxGroup = 32;    // query heads per KV head handled by one attention CTA

// ---- top-k radix select: 32-bit orderable keys, digits of 12 + 12 + 8 bits ----
constexpr int kBins1 = 4096;
constexpr int kBins2 = 4096;
constexpr int kBins3 = 256;
constexpr int kCandCap = 4096;  // boundary-bin candidates finished in shared memory

enum SelectMode : int {
    kSelUndecided = 0,  // more digits needed
    kSelAll = 1,        // n_c <= top_k: every candidate
    kSelPrefix = 2,     // keys whose top `nbits` exceed or equal `prefix`
    kSelTies = 3,       // keys above `prefix` (full 32 bits) and the first `need` equal ones
};

// Per-query control block of the decode select, zeroed before every select.
struct TopkCtrl {
    unsigned hist1[kBins1];
    unsigned done[4];      // CTA completion counters of the passes
    unsigned nsel;         // entries appended to the unordered list
    unsigned prefix;       // resolved high bits of the threshold key
    int nbits;             // how many high bits are resolved
    int need;              // entries still to take from keys equal to `prefix`
    int mode;              // SelectMode
    int n_cand;            // n_c of the query (after the max_blocks cut)
    unsigned bin_count;    // keys in the bin of the last resolved digit
    unsigned ncand;        // entries appended to the candidate list
    unsigned pad[4];
};
static_assert(sizeof(TopkCtrl) % 64 == 0, "TopkCtrl keeps 64-byte alignment");

// fp32 -> unsigned key with the same order (larger float -> larger key); -0 maps to +0.
__device__ __forceinline__ unsigned orderable_key(float f)
{
    unsigned u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ void set_status(unsigned* status, unsigned bit)
{
    if (status) atomicOr(status, bit);
}

// Programmatic dependent launch.  A kernel launched with launch_k(..., pdl = true)
// may start while the previous kernel in the stream is still running; before
// griddep_wait() it may only read inputs that were complete before the layer call
// began.  Every kernel calls griddep_launch_dependents() only after its own
// griddep_wait(), so a dependent never overlaps anything older than its direct
// predecessor.  Without a programmatic dependency both are no-ops.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
                            Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = pdl ? attr : nullptr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// two bf16 packed in a 32-bit word -> two fp32 (exact)
__device__ __forceinline__ float bf16lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf16hi(uint32_t x) { return __uint_as_float(x & 0xFFFF0000u); }

// ---- workspace layout ----
struct WsLayout {
    size_t status = 0;     // u32 status word (first 256 bytes)
    size_t ctrl = 0;       // TopkCtrl[n_q] then attention counters u32[n_q * n_kv_heads]
    size_t ctrl_bytes = 0; // bytes zeroed at the start of each select/attention
    size_t attn_cnt = 0;   // offset of the attention split counters (inside ctrl)
    size_t cand = 0;       // u64 [rows][kCandCap] boundary-bin candidates (key << 32 | block)
    size_t tmp = 0;        // i32 [rows][top_k] unordered winners
    size_t scores = 0;     // f32 [n_rows][ld] decode score rows
    int64_t score_ld = 0;
    int32_t score_rows = 0;
    size_t sel = 0;        // i32 [n_q][top_k] + i32 [n_q] when the caller passes none
    size_t partial = 0;    // f32 split-K partials of the decode attention
    // prefill (tensor-core) select
    size_t pf_cand = 0;    // u64 [n_q][2 * pf_split][seg_cap] admitted (key << 32 | block)
    size_t pf_cnt = 0;     // u32 [n_q][2 * pf_split]
    size_t pf_theta = 0;   // u32 [n_q] shared thresholds (zeroed per call)
    size_t pf_work = 0;    // i32 [1 + n_q] fallback worklist (count zeroed per call)
    size_t pf_shist = 0;   // u32 [n_q][2][65] sampled score histograms
    size_t pf_scratch = 0; // f32 [pf_fb_ctas][max_blocks]
    size_t qpos_loc = 0;   // i32 [n_q] positions inside a context shard
    int pf_split = 0;
    int pf_fb_ctas = 0;
    size_t total = 0;
    int n_chunks = 0;
    int chunk = 0;
};

// ---- host-side argument checks shared by every entry point (api.cu) ----
// Pointer non-null and 16-byte aligned.
bool aligned16(const void* p);
// The dims every call needs: sizes, fixed method parameters, supported head layout.
int check_dims(const qsa_dims* d);
// Query count and candidate-block bound of a call.
int check_rows(const qsa_dims* d, int32_t n_q, int64_t max_blocks);
// Draft-query groups sharing one selection: group_q >= 1 divides n_q, rows per CTA <= 32.
int check_groups(const qsa_dims* d, int32_t n_q, int32_t group_q);
// Paged K/V (page_table may be NULL: dense caches).
int check_pages(const qsa_dims* d, const int32_t* page_table, int32_t page_tokens, int64_t n_pages);

// Chunk of candidate blocks one CTA of the decode scoring/select passes handles.
int select_chunk(int64_t max_blocks, int32_t n_rows);
WsLayout plan_workspace(const qsa_dims& d, int32_t n_q, int64_t max_blocks, int32_t mode);

// ---- launchers (return cudaGetLastError()) ----
// Pool the blocks completed by the append (max_new_tokens may be 0) and, in the
// same launch, zero `zero_bytes` (a multiple of 16) at `zero` (may be null).
cudaError_t launch_pool(const qsa_dims& d, const void* idx_k, void* pooled, const int32_t* len_before,
                        const int32_t* len_after, int32_t max_new_tokens, void* zero, size_t zero_bytes,
                        unsigned* status, cudaStream_t st);

// Scores for rows [row0, row0 + n_rows) (query i = row0 + r).  With ctrl != nullptr
// also builds the digit-1 histogram; then, with sel_idx != nullptr (needs
// max_blocks <= 16,384) the last CTA of each row selects the row completely,
// otherwise it resolves digit 1 for launch_topk.
// Row r's query indexer inputs are q_idx[row0 + r], w[row0 + r]; its sequence and
// position are q_seq / q_pos[(row0 + r) * pos_stride] (pos_stride > 1: one selection
// per group of draft queries, made for the group's first query).
cudaError_t launch_score_decode(const qsa_dims& d, const void* q_idx, const float* w, const void* pooled,
                                const int32_t* q_seq, const int32_t* q_pos, int32_t row0, int32_t n_rows,
                                int64_t max_blocks, float* scores, int64_t ld, int chunk, TopkCtrl* ctrl,
                                int32_t* sel_idx, int32_t* sel_cnt, unsigned* status, cudaStream_t st,
                                bool pdl = false, int pos_stride = 1);
// Largest max_blocks for which launch_score_decode can finish the select itself.
constexpr int64_t kScoreFinishMaxBlocks = 16384;

// Radix select over score rows [0, n_rows) (query i = row0 + r).  If `hist_done`
// the digit-1 histogram was built by the scoring kernel.
cudaError_t launch_topk(const float* scores, int64_t ld, const int32_t* q_pos, int32_t row0, int32_t n_rows,
                        int64_t max_blocks, int64_t kv_capacity, int bs, int top_k, int chunk, int n_chunks,
                        TopkCtrl* ctrl,
                        unsigned long long* cand, int32_t* tmp, int32_t* sel_idx, int32_t* sel_cnt, bool hist_done,
                        unsigned* status, cudaStream_t st, bool pdl = false);

// Prefill chunk (queries of one sequence per 128-row tile): tcgen05 scoring with
// streaming admission, exact finishing select, fallback for unsettled rows.
int prefill_splits(int32_t n_q, int64_t max_blocks);
int prefill_seg_cap();
int prefill_segments(int n_split);  // admission segments per query row
int prefill_shist_words(int n_split);
bool prefill_sampled(const qsa_dims& d, int64_t max_blocks);
cudaError_t launch_prefill_select(const qsa_dims& d, const void* q_idx, const float* w, const void* pooled,
                                  const int32_t* q_seq, const int32_t* q_pos, int32_t n_q, int64_t max_blocks,
                                  int n_split, unsigned long long* cand, unsigned* cand_cnt, unsigned* theta_g,
                                  uint32_t* shist, int32_t* worklist, float* scratch, int n_fallback_ctas,
                                  int32_t* sel_idx, int32_t* sel_cnt, unsigned* status, cudaStream_t st);

// Gathered attention (attn.cu): groups of `group_q` queries sharing one selection
// row, optional paged K/V.  Few (group, KV head) pairs split their block lists; the
// splits merge in a thread-block cluster when allow_cluster and the device can hold
// every cluster at once, else through `partial` / `counters` (counters zeroed by the
// caller).  Many pairs run one CTA per pair, two CTAs per SM.
int attn_split_bound(int64_t pairs);
// The launch shape of launch_sparse_attn for n_groups groups (host arithmetic only).
bool describe_sparse_attn(const qsa_dims& d, int64_t n_groups, int group_q, bool allow_cluster, int* n_split,
                          int* stages, int* threads, int* smem, int64_t* ctas, int* cluster, int* rows);
size_t attn_partial_bytes();  // bytes of `partial` any launch needs
size_t attn_counter_bytes();  // bytes of `counters` any launch needs (one word per split pair)
cudaError_t launch_sparse_attn(const qsa_dims& d, const void* q, const void* k_cache, const void* v_cache,
                               const int32_t* q_seq, const int32_t* q_pos, const int32_t* sel_idx,
                               const int32_t* sel_cnt, const int32_t* page_table, int page_tokens, int64_t n_pages,
                               int64_t n_groups, int group_q, void* out, float* partial, unsigned* counters,
                               unsigned* status, cudaStream_t st, bool pdl, bool allow_cluster,
                               bool counters_zeroed, float* part_out = nullptr);

// Context-parallel steps (cp.cu).
size_t cp_partial_row_floats();
cudaError_t launch_cp_local_pos(const int32_t* q_pos, int32_t n_q, int64_t tok_lo, int64_t cap_loc, int32_t* pos_loc,
                                cudaStream_t st);
cudaError_t launch_cp_keys(const float* scores, int64_t ld, const int32_t* sel, const int32_t* cnt, int32_t n_q,
                           int64_t blk_lo, unsigned long long* keys, int32_t* key_cnt, cudaStream_t st);
cudaError_t launch_cp_merge(const unsigned long long* keys_all, const int32_t* cnt_all, int n_ranks, int32_t n_q,
                            int top_k, int64_t blk_lo, int64_t n_local, int32_t* sel_local, int32_t* cnt_local,
                            int32_t* sel_global, int32_t* cnt_global, cudaStream_t st);
cudaError_t launch_cp_combine(const float* parts, int n_ranks, int64_t rows, void* out, cudaStream_t st);

}  // namespace qsa
