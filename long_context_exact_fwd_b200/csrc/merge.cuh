// Log-sum-exp merge of normalised partial attention outputs (HBM-bound).
//
// Pages: "精读笔记 · Ring Attention with Blockwise Transformers for Near-Infinite Context",
// §3.1 (blocks combined in any order once their statistics are rescaled); "RingAttention
// large-context attention", 架构与算法 (partial outputs aggregated into the final output --
// read as the LSE-weighted combination, a plain sum of normalised partials is not attention):
//   lse = log sum_p exp(lse_p),  o = sum_p exp(lse_p - lse) o_p,
// a partial with lse_p = -inf weighs 0; all -inf gives o = 0, lse = -inf.
//
// One warp per row: each lane owns float4 column groups, so every partial row is read as
// one fully coalesced 16-byte-per-lane sweep; the per-partial weights are computed once per
// lane from the P log-sum-exps (a few bytes, cached).
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

namespace ra {
namespace merge {

constexpr int WARPS = 8;

__device__ __forceinline__ void store4(float* dst, float4 v) { *reinterpret_cast<float4*>(dst) = v; }
__device__ __forceinline__ void store4(__nv_bfloat16* dst, float4 v) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(dst) = u;
}

template <typename OutT>
__global__ void __launch_bounds__(WARPS * 32)
    merge_kernel(const float* __restrict__ o_parts, const float* __restrict__ lse_parts, int P,
                 OutT* __restrict__ o, float* __restrict__ lse, long long rows, int Dh) {
  const int lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * WARPS + (threadIdx.x >> 5);
  if (row >= rows) return;
  float m = -INFINITY;
  for (int p = 0; p < P; ++p) m = fmaxf(m, __ldg(lse_parts + p * rows + row));
  const int groups = Dh >> 2;
  if (m == -INFINITY) {
    for (int g = lane; g < groups; g += 32) store4(o + row * Dh + 4 * g, make_float4(0.f, 0.f, 0.f, 0.f));
    if (lane == 0) lse[row] = -INFINITY;
    return;
  }
  float z = 0.f;
  for (int p = 0; p < P; ++p) z += expf(__ldg(lse_parts + p * rows + row) - m);
  const float lse_row = m + logf(z);
  for (int g = lane; g < groups; g += 32) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int p = 0; p < P; ++p) {
      const float w = expf(__ldg(lse_parts + p * rows + row) - lse_row);
      const float4 x = __ldg(reinterpret_cast<const float4*>(o_parts + (p * rows + row) * Dh) + g);
      acc.x = fmaf(w, x.x, acc.x);
      acc.y = fmaf(w, x.y, acc.y);
      acc.z = fmaf(w, x.z, acc.z);
      acc.w = fmaf(w, x.w, acc.w);
    }
    store4(o + row * Dh + 4 * g, acc);
  }
  if (lane == 0) lse[row] = lse_row;
}

}  // namespace merge
}  // namespace ra
