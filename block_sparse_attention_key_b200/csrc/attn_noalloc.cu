// Gathered attention for callers that cannot allocate device memory.
//
// qsa_sparse_attn needs a caller workspace for its split-K partials and
// completion counters.  Some callers have no way to provide one: code running
// under an allocator that forbids new device allocations (a serving engine that
// reserved all of HBM for its KV cache up front, a CUDA-graph replay path whose
// memory plan is frozen), or plain C hosts that only hand over the tensors they
// already own.  This entry point runs the same attention kernel with its
// scratch taken from a fixed array compiled into the library instead.
//
// The scratch is a file-scope __device__ array of kScratchBytes.  Every GPU that
// loads this library holds that much memory until the process exits.  On the
// host the array's name is only a stand-in, not a device address, so the first
// call on each device (with that device current) looks the address up with
// cudaGetSymbolAddress, and every later call made outside stream capture looks
// it up again; the first call on each device should therefore come before any
// stream capture.  All calls share the one array and it keeps the previous
// call's contents: the completion counters are cleared at the start of
// every call, and calls whose executions overlap on the GPU (for example on two
// streams) race on it.  Nothing here calls cudaMalloc, cudaFree or any other
// allocating routine.

#include <mutex>

#include "qsa_internal.cuh"

namespace qsa {

namespace {

constexpr size_t kScratchBytes = 16u << 20;  // 16 MiB: counters + split partials
constexpr size_t kCounterAlign = 256;
constexpr int kMaxDevices = 128;

__device__ __align__(256) unsigned char g_attn_scratch[kScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_attn_scratch on the current device.  Looked up afresh on
// every call made outside stream capture (so a device reset, which rebuilds the
// context and may move the array, never leaves a stale address in use); a call
// made while `st` is capturing reuses the address of the last uncaptured call on
// this device, and fails if there was none.
cudaError_t scratch_address(cudaStream_t st, void** out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    e = cudaStreamIsCapturing(st, &cap);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (cap == cudaStreamCaptureStatusNone) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_attn_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    } else if (!g_scratch_ptr[dev]) {
        return cudaErrorStreamCaptureUnsupported;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

}  // namespace qsa

using namespace qsa;

extern "C" int qsa_sparse_attn_noalloc(const qsa_dims* dims, const void* q, const void* k_cache,
                                       const void* v_cache, const int32_t* q_seq, const int32_t* q_pos,
                                       const int32_t* sel_idx, const int32_t* sel_cnt, int32_t n_q, void* out,
                                       void* stream)
{
    // same argument rules as qsa_sparse_attn (the shared checks), minus the workspace
    int rc = check_dims(dims);
    if (rc != QSA_OK) return rc;
    if ((rc = check_rows(dims, n_q, 0)) != QSA_OK) return rc;
    if (n_q == 0) return QSA_OK;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(q_seq) || !aligned16(q_pos) ||
        !aligned16(sel_idx) || !aligned16(sel_cnt) || !aligned16(out))
        return QSA_ERR_INVALID_ARG;

    const int64_t pairs = (int64_t)n_q * dims->n_kv_heads;
    const int n_split = attn_split_bound(pairs);
    const size_t counter_bytes = ((size_t)pairs * 4 + kCounterAlign - 1) / kCounterAlign * kCounterAlign;
    const size_t partial_bytes = n_split > 1 ? attn_partial_bytes() : 0;
    if (counter_bytes + partial_bytes > kScratchBytes) return QSA_ERR_WORKSPACE_TOO_SMALL;

    cudaStream_t st = (cudaStream_t)stream;
    void* base = nullptr;
    if (scratch_address(st, &base) != cudaSuccess) return QSA_ERR_CUDA;
    unsigned* counters = (unsigned*)base;
    float* partial = (float*)((char*)base + counter_bytes);
    if (n_split > 1 && cudaMemsetAsync(counters, 0, (size_t)pairs * 4, st) != cudaSuccess) return QSA_ERR_CUDA;
    // no status word in this variant: out-of-range indices are still skipped, just not
    // reported; split partials always meet through the scratch array
    const cudaError_t e = launch_sparse_attn(*dims, q, k_cache, v_cache, q_seq, q_pos, sel_idx, sel_cnt, nullptr, 0,
                                             0, n_q, 1, out, partial, counters, nullptr, st, false, false, true);
    return e == cudaSuccess ? QSA_OK : QSA_ERR_CUDA;
}
