// Device twin of qsa_synth/gen.py: fills the synthetic QSA inputs in place on the
// GPU, bit-identical to the host generator (same SplitMix64 streams, same value
// recipes).  Input generation only: none of the layer's arithmetic is here.
//
// SplitMix64 (Steele, Lea, Flood 2014; Vigna's finaliser constants): output i of
// a stream keyed `key` is mix(key + (i + 1) * GAMMA).
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

__device__ __forceinline__ uint64_t mix64(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

__device__ __forceinline__ uint64_t draw(uint64_t key, uint64_t idx) { return mix64(key + (idx + 1) * kGamma); }

__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f)
{
    const uint32_t b = __float_as_uint(f);
    return (uint16_t)((b + 0x7FFFu + ((b >> 16) & 1u)) >> 16);
}

// Irwin-Hall(4) of 16-bit uniforms, centred, scaled to unit variance; fp64 -> fp32 -> bf16
__device__ __forceinline__ uint16_t unit_normal_bf16(uint64_t r)
{
    const uint64_t s = (r & 0xFFFF) + ((r >> 16) & 0xFFFF) + ((r >> 32) & 0xFFFF) + ((r >> 48) & 0xFFFF);
    double x = __ddiv_rn(__dadd_rn((double)s, 2.0), 65536.0);
    x = __dmul_rn(__dadd_rn(x, -2.0), 1.7320508075688772);
    return f32_to_bf16_rne(__double2float_rn(x));
}

__device__ __forceinline__ int64_t uniform_int(uint64_t r, int lo, int hi)
{
    const uint64_t n = (uint64_t)(hi - lo + 1);
    return (int64_t)(((r >> 32) * n) >> 32) + lo;
}

__device__ __forceinline__ uint16_t small_int_bf16(int64_t v)
{
    return (uint16_t)(__float_as_uint((float)v) >> 16);
}

// K or V cache [B][H][T][D] (head-major), logical coordinate (s, g, t, d)
__global__ void k_fill_kv(uint16_t* dst, int64_t B, int64_t H, int64_t T, int64_t D, uint64_t key)
{
    const int64_t n = B * H * T * D;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t d = e % D, t = (e / D) % T, g = (e / (D * T)) % H, s = e / (D * T * H);
        const uint64_t c = (((((uint64_t)s << 8) | (uint64_t)g) << 32 | (uint64_t)t) << 8) | (uint64_t)d;
        dst[e] = unit_normal_bf16(draw(key, c));
    }
}

// indexer keys [B][T][Di], logical coordinate (s, t, d), integers on [lo, hi]
__global__ void k_fill_idxk(uint16_t* dst, int64_t B, int64_t T, int64_t Di, uint64_t key, int lo, int hi)
{
    const int64_t n = B * T * Di;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t d = e % Di, t = (e / Di) % T, s = e / (Di * T);
        const uint64_t c = ((((uint64_t)s << 32) | (uint64_t)t) << 8) | (uint64_t)d;
        dst[e] = small_int_bf16(uniform_int(draw(key, c), lo, hi));
    }
}

// per-query rows [n][H][D] with query ids qid0 + row; normal (kind 0) or integers (kind 1)
__global__ void k_fill_query(uint16_t* dst, int64_t n_rows, int64_t H, int64_t D, int64_t qid0, uint64_t key,
                             int kind, int lo, int hi)
{
    const int64_t n = n_rows * H * D;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t d = e % D, h = (e / D) % H, i = e / (D * H);
        const uint64_t c = ((uint64_t)(qid0 + i) << 16) | ((uint64_t)h << 8) | (uint64_t)d;
        const uint64_t r = draw(key, c);
        dst[e] = kind == 0 ? unit_normal_bf16(r) : small_int_bf16(uniform_int(r, lo, hi));
    }
}

// per-query head weights [n][H] (float), integers on [lo, hi]
__global__ void k_fill_weights(float* dst, int64_t n_rows, int64_t H, int64_t qid0, uint64_t key, int lo, int hi)
{
    const int64_t n = n_rows * H;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t h = e % H, i = e / H;
        const uint64_t c = ((uint64_t)(qid0 + i) << 8) | (uint64_t)h;
        dst[e] = (float)uniform_int(draw(key, c), lo, hi);
    }
}

unsigned grid_for(int64_t n) { return (unsigned)(n / 256 + 1 < 148 * 64 ? n / 256 + 1 : 148 * 64); }

}  // namespace

extern "C" {

int synth_fill_kv(void* dst, int64_t B, int64_t H, int64_t T, int64_t D, uint64_t key, void* stream)
{
    k_fill_kv<<<grid_for(B * H * T * D), 256, 0, (cudaStream_t)stream>>>((uint16_t*)dst, B, H, T, D, key);
    return (int)cudaGetLastError();
}

int synth_fill_idxk(void* dst, int64_t B, int64_t T, int64_t Di, uint64_t key, int lo, int hi, void* stream)
{
    k_fill_idxk<<<grid_for(B * T * Di), 256, 0, (cudaStream_t)stream>>>((uint16_t*)dst, B, T, Di, key, lo, hi);
    return (int)cudaGetLastError();
}

int synth_fill_query(void* dst, int64_t n_rows, int64_t H, int64_t D, int64_t qid0, uint64_t key, int kind,
                     int lo, int hi, void* stream)
{
    k_fill_query<<<grid_for(n_rows * H * D), 256, 0, (cudaStream_t)stream>>>((uint16_t*)dst, n_rows, H, D, qid0,
                                                                              key, kind, lo, hi);
    return (int)cudaGetLastError();
}

int synth_fill_weights(void* dst, int64_t n_rows, int64_t H, int64_t qid0, uint64_t key, int lo, int hi,
                       void* stream)
{
    k_fill_weights<<<grid_for(n_rows * H), 256, 0, (cudaStream_t)stream>>>((float*)dst, n_rows, H, qid0, key, lo,
                                                                           hi);
    return (int)cudaGetLastError();
}

}  // extern "C"
