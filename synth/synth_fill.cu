// synth_fill.cu -- device copy of the seeded input generator defined in
// synth/__init__.py (SplitMix64 output function of Steele, Lea & Flood 2014;
// Irwin-Hall sum of four 16-bit fields; one IEEE double multiply; round to
// float32 then bf16, both to nearest even).  It draws numbers only; it holds
// none of the attention arithmetic.  Bit-identical to the numpy generator.
#include <cuda_bf16.h>
#include <stdint.h>

#define SYNTH_API extern "C" __attribute__((visibility("default")))

namespace {
constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;
constexpr double kInvSd = 2.6428997921303014e-05;

__host__ __device__ inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__host__ __device__ inline uint64_t stream_key(uint64_t seed, int tensor, int64_t request) {
  const uint64_t k0 = mix64(seed + kGamma * (uint64_t)(1 + tensor));
  return mix64(k0 + kGamma * (uint64_t)(1 + request));
}

__device__ inline uint16_t draw(uint64_t key, uint64_t e, double amp) {
  const uint64_t x = mix64(key + kGamma * (e + 1));
  const int64_t s = (int64_t)(x & 0xFFFF) + (int64_t)((x >> 16) & 0xFFFF) + (int64_t)((x >> 32) & 0xFFFF) +
                    (int64_t)(x >> 48);
  const double z = (double)(s - 131070) * kInvSd;
  const double v = __dmul_rn(z, amp);
  const float f = __double2float_rn(v);
  const __nv_bfloat16 h = __float2bfloat16_rn(f);
  return *reinterpret_cast<const uint16_t*>(&h);
}

// Rows of `row_elems` elements for requests concatenated by cu_seqlens.
// GQA (kind 0): row [2][Hkv][d]: K from tensor 2, V from tensor 3, e = (t*Hkv + h)*d + k.
// MLA (kind 1): row [d]: tensor 4, e = t*d + k.
// Query (kind 2): rows are (request, head) pairs [B*H][d]: tensor 1, e = h*d + k.
__global__ void fill_kernel(uint16_t* dst, const int64_t* cu_seqlens, int B, int kind, int Hkv, int d,
                            uint64_t seed, double amp, int64_t total_rows) {
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int row_elems = kind == 0 ? 2 * Hkv * d : d;
  for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < total_rows; r += nwarps) {
    int64_t b, t;
    if (kind == 2) {
      b = r / Hkv;  // Hkv carries the number of heads for queries
      t = r - b * Hkv;
    } else {
      int lo = 0, hi = B - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (cu_seqlens[mid] <= r) lo = mid; else hi = mid - 1;
      }
      b = lo;
      t = r - cu_seqlens[b];
    }
    uint16_t* out = dst + r * row_elems;
    if (kind == 0) {
      const uint64_t kk = stream_key(seed, 2, b), kv = stream_key(seed, 3, b);
      for (int i = lane; i < row_elems; i += 32) {
        const int half = i / (Hkv * d), rem = i - half * Hkv * d;  // rem = h*d + k
        out[i] = draw(half == 0 ? kk : kv, (uint64_t)(t * Hkv * d + rem), amp);
      }
    } else if (kind == 1) {
      const uint64_t k = stream_key(seed, 4, b);
      for (int i = lane; i < row_elems; i += 32) out[i] = draw(k, (uint64_t)(t * d + i), amp);
    } else {
      const uint64_t k = stream_key(seed, 1, b);
      for (int i = lane; i < row_elems; i += 32) out[i] = draw(k, (uint64_t)(t * d + i), amp);
    }
  }
}
}  // namespace

SYNTH_API int synth_fill(void* dst, const int64_t* cu_seqlens, int B, int kind, int Hkv, int d, uint64_t seed,
                         double amp, int64_t total_rows, int sm_count, void* stream) {
  if (total_rows <= 0) return 0;
  fill_kernel<<<sm_count * 8, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint16_t*>(dst), cu_seqlens, B, kind, Hkv, d, seed, amp, total_rows);
  return cudaGetLastError() == cudaSuccess ? 0 : 1;
}
