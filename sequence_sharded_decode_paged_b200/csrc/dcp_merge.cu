// dcp_merge.cu -- on-device LSE merge of D partial attention outputs.
//
// "Efficient Decode Context Parallelism with vLLM for Long Context
// Workloads", A2 方法细节: the partial outputs O_i of the shards are
// re-weighted by their log-sum-exp values and summed,
//     O = sum_i exp(LSE_i) / sum_j exp(LSE_j) * O_i,
// which on one GPU replaces the AllGather + ReduceScatter exchange.  It is
// evaluated against the largest LSE so that no exponential overflows
// (the local-max form of "vLLM长序列推理优化：DCP切分KV Cache原理与实战" §2.3).
//
// Bandwidth bound: D*rows*(d_v+1)*4 bytes read, rows*(d_v+1)*4 written.
// Each thread produces one float4 of the output and issues the D float4
// loads of its inputs back to back; the D LSE values of its row come from
// L1 (they are shared by the d_v/4 threads of the row).
#include "dcp_device.cuh"
#include "dcp_internal.h"

namespace dcp {

struct MergeParams {
  const float4* O[kMaxShards];
  const float* LSE[kMaxShards];
  float4* out;
  float* lse_out;
  int D;
  int rows;
  int vec_per_row;  // d_v / 4
};

template <int DMAX>
__global__ void __launch_bounds__(256) lse_merge_kernel(const __grid_constant__ MergeParams p) {
  const long total = (long)p.rows * p.vec_per_row;
  for (long idx = (long)blockIdx.x * blockDim.x + threadIdx.x; idx < total; idx += (long)gridDim.x * blockDim.x) {
    const int row = (int)(idx / p.vec_per_row);
    const int vec = (int)(idx - (long)row * p.vec_per_row);
    float lse[DMAX];
    float4 part[DMAX];
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < DMAX; ++i) {
      if (i < p.D) {
        lse[i] = __ldg(p.LSE[i] + row);
        part[i] = __ldcs(p.O[i] + idx);
        mx = fmaxf(mx, lse[i]);
      }
    }
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float wsum = 0.f;
    if (mx != -INFINITY) {
#pragma unroll
      for (int i = 0; i < DMAX; ++i) {
        if (i < p.D) {
          const float w = lse[i] == -INFINITY ? 0.f : expf(lse[i] - mx);
          wsum += w;
          acc.x += w * part[i].x;
          acc.y += w * part[i].y;
          acc.z += w * part[i].z;
          acc.w += w * part[i].w;
        }
      }
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    __stcs(p.out + idx, make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv));
    if (p.lse_out != nullptr && vec == 0) p.lse_out[row] = wsum > 0.f ? mx + logf(wsum) : -INFINITY;
  }
}

dcp_status launch_lse_merge(const float* const* O_parts, const float* const* LSE_parts, int D, int rows, int d_v,
                            float* O, float* LSE_out, cudaStream_t st) {
  MergeParams p;
  memset(&p, 0, sizeof(p));
  for (int i = 0; i < D; ++i) {
    p.O[i] = reinterpret_cast<const float4*>(O_parts[i]);
    p.LSE[i] = LSE_parts[i];
  }
  p.out = reinterpret_cast<float4*>(O);
  p.lse_out = LSE_out;
  p.D = D;
  p.rows = rows;
  p.vec_per_row = d_v / 4;
  const long total = (long)rows * p.vec_per_row;
  if (total == 0) return DCP_OK;
  const int threads = 256;
  long blocks = (total + threads - 1) / threads;
  const long cap = (long)device_sm_count() * 8;
  if (blocks > cap) blocks = cap;
  if (D <= 2)
    lse_merge_kernel<2><<<(unsigned)blocks, threads, 0, st>>>(p);
  else if (D <= 4)
    lse_merge_kernel<4><<<(unsigned)blocks, threads, 0, st>>>(p);
  else if (D <= 8)
    lse_merge_kernel<8><<<(unsigned)blocks, threads, 0, st>>>(p);
  else
    lse_merge_kernel<16><<<(unsigned)blocks, threads, 0, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? DCP_OK : DCP_ERR_CUDA;
}

}  // namespace dcp
