// Float32 forward on CUDA cores: one warp per query row, lanes split the head dimension.
//
// Same method as the bf16 kernel (pages: "精读笔记 · Ring Attention with Blockwise
// Transformers for Near-Infinite Context", §3.1 online-softmax combination, §3.5 ring order),
// without tensor cores: every score, exponential and accumulation is float32, so the result
// tracks the exact definition to ~1e-6.  Used for float32 inputs (e.g. the 256-token
// exactness workload); it is not a throughput path.
#pragma once
#include <cstdint>

namespace ra {
namespace f32 {

constexpr int WARPS = 8;
constexpr int MAX_VPL = 8;   // values per lane: Dh <= 256

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

template <int VPL>
__global__ void __launch_bounds__(WARPS * 32)
    fwd_f32_kernel(const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
                   float* __restrict__ o, float* __restrict__ lse, long long rows, int S, int Dh, int D, int causal,
                   float scale) {
  const int lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * WARPS + (threadIdx.x >> 5);
  if (row >= rows) return;  // warp-uniform
  const long long bh = row / S;
  const int i = static_cast<int>(row - bh * S);
  const float* kb = k + bh * S * Dh;
  const float* vb = v + bh * S * Dh;
  float qv[VPL], acc[VPL];
#pragma unroll
  for (int j = 0; j < VPL; ++j) {
    const int d = lane + 32 * j;
    qv[j] = d < Dh ? q[row * Dh + d] : 0.f;
    acc[j] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const int c = S / D;
  const int r = i / c;
  for (int t = 0; t < D; ++t) {              // ring step t: block (r - t) mod D
    const int blk = ((r - t) % D + D) % D;
    const int kbeg = blk * c;
    int kend = kbeg + c;
    if (causal && kend > i + 1) kend = i + 1;
    for (int kj = kbeg; kj < kend; ++kj) {
      float part = 0.f;
#pragma unroll
      for (int j = 0; j < VPL; ++j) {
        const int d = lane + 32 * j;
        if (d < Dh) part = fmaf(qv[j], kb[static_cast<long long>(kj) * Dh + d], part);
      }
      const float s = warp_sum(part) * scale;
      float a, pw;
      if (s > m) {              // new running max: rescale what was accumulated
        a = (m == -INFINITY) ? 0.f : expf(m - s);
        pw = 1.f;
        m = s;
      } else {
        a = 1.f;
        pw = expf(s - m);
      }
      l = fmaf(l, a, pw);
#pragma unroll
      for (int j = 0; j < VPL; ++j) {
        const int d = lane + 32 * j;
        const float vv = d < Dh ? vb[static_cast<long long>(kj) * Dh + d] : 0.f;
        acc[j] = fmaf(acc[j], a, pw * vv);
      }
    }
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
  for (int j = 0; j < VPL; ++j) {
    const int d = lane + 32 * j;
    if (d < Dh) o[row * Dh + d] = acc[j] * inv;
  }
  if (lane == 0) lse[row] = l > 0.f ? m + logf(l) : -INFINITY;
}

}  // namespace f32
}  // namespace ra
