// Log-sum-exp merge of normalised partial attention outputs (HBM-bound).
//
// Pages: "精读笔记 · Ring Attention with Blockwise Transformers for Near-Infinite Context",
// §3.1 (blocks combined in any order once their statistics are rescaled); "RingAttention
// large-context attention", 架构与算法 (partial outputs aggregated into the final output --
// read as the LSE-weighted combination, a plain sum of normalised partials is not attention):
//   lse = log sum_p exp(lse_p),  o = sum_p exp(lse_p - lse) o_p,
// a partial with lse_p = -inf weighs 0; all -inf gives o = 0, lse = -inf.
//
// One warp per row at a time (grid-stride over rows): each lane owns float4 column groups, so
// every partial row is read as one coalesced 16-byte-per-lane sweep.  The partials are folded
// in online, four at a time -- running max m, rescaled sum z and accumulator -- with the four
// log-sum-exps and the four float4 rows of a chunk loaded together, so a row costs one
// memory round trip per four partials instead of a round trip for the weights followed by one
// per partial:  m' = max(m, lse_p..), acc = acc e^(m-m') + sum_p e^(lse_p-m') o_p,
// z = z e^(m-m') + sum_p e^(lse_p-m');  o = acc / z,  lse = m + log z.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

namespace ra {
namespace merge {

constexpr int WARPS = 8;
constexpr int CHUNK = 4;          // partials loaded together
constexpr int BLOCKS_PER_SM = 8;  // grid cap per SM (4 blocks are resident at 64 registers; the rest queue)

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
  const int groups = Dh >> 2;
  const long long n_warps = static_cast<long long>(gridDim.x) * WARPS;
  const float4* parts4 = reinterpret_cast<const float4*>(o_parts);
  for (long long row = static_cast<long long>(blockIdx.x) * WARPS + (threadIdx.x >> 5); row < rows; row += n_warps) {
    float m = -INFINITY, z = 0.f;
    for (int g = lane; g < groups; g += 32) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      m = -INFINITY;
      z = 0.f;
      for (int p0 = 0; p0 < P; p0 += CHUNK) {
        float l[CHUNK];
        float4 x[CHUNK];
#pragma unroll
        for (int j = 0; j < CHUNK; ++j) {
          const int pp = p0 + j;
          if (pp < P) {
            const long long pr = static_cast<long long>(pp) * rows + row;
            l[j] = __ldg(lse_parts + pr);
            x[j] = __ldg(parts4 + pr * groups + g);
          } else {
            l[j] = -INFINITY;
            x[j] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
        const float mn = fmaxf(fmaxf(m, fmaxf(l[0], l[1])), fmaxf(l[2], l[3]));
        if (mn == -INFINITY) continue;                    // nothing visible so far
        const float sc = (m == -INFINITY) ? 0.f : expf(m - mn);
        acc.x *= sc;
        acc.y *= sc;
        acc.z *= sc;
        acc.w *= sc;
        z *= sc;
#pragma unroll
        for (int j = 0; j < CHUNK; ++j) {
          if (l[j] == -INFINITY) continue;   // a -inf partial weighs 0, whatever its o holds
          const float w = expf(l[j] - mn);
          acc.x = fmaf(w, x[j].x, acc.x);
          acc.y = fmaf(w, x[j].y, acc.y);
          acc.z = fmaf(w, x[j].z, acc.z);
          acc.w = fmaf(w, x[j].w, acc.w);
          z += w;
        }
        m = mn;
      }
      const float inv = (m == -INFINITY) ? 0.f : 1.f / z;
      store4(o + row * Dh + 4 * g, make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv));
    }
    if (lane == 0) lse[row] = (m == -INFINITY) ? -INFINITY : m + logf(z);
  }
}

}  // namespace merge
}  // namespace ra
