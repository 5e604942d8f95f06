// Blockwise feedforward after attention, for sm_100a: a persistent TMA + tcgen05 GEMM with a
// fused bias / GELU epilogue, run on one ring block of c tokens at a time.
//
// Page "精读笔记 · Ring Attention with Blockwise Transformers for Near-Infinite Context", §2.2
// (BPT): the feedforward of each attention sub-layer is computed block by block, so its largest
// activation is one block's hidden layer instead of the whole sequence's (2bsh instead of 8bsh
// bytes); §3.5 Algorithm 1: per layer each host's block goes through attention, then the
// feedforward.  Y = gelu(X W1^T + b1) W2^T + b2 with X the block's attention output, heads side
// by side per token; GELU in its exact form x Phi(x) (the pages name no activation).
//
// One kernel computes C[m, n] = epi(sum_k A[m, k] B[n, k] + bias[n]) for one block:
//   GEMM 1: A = the attention output O [B][H][S][Dh] read in place (token rows of the block,
//           K index = head * Dh + d), B = W1 [f][h], epi = GELU, C = Z [B][c][f] (workspace);
//   GEMM 2: A = Z, B = W2 [h][f], epi = identity, C = Y [B][S][h] rows of the block.
// Both operands are K-major and arrive by 3-D TMA tile loads (128-byte swizzle, no multicast);
// an A tile never crosses a batch entry, and rows past the block are loaded but not stored.
//
// CTA (256 threads, persistent, tiles t = blockIdx.x + i * gridDim.x, M-tiles fastest):
//   warps 0-3  epilogue: thread = output row = TMEM lane; TMEM -> registers -> bias, GELU ->
//              bf16 -> 16-byte global stores, 32 columns at a time;
//   warp 4     TMA producer: per 64-wide K step, A 128 x 64 and B 256 x 64 into a 4-stage ring;
//   warp 5     TMEM allocator + tcgen05.mma issuer (M = 128, N = 256, K = 16).
// TMEM (512 columns): two 128 x 256 fp32 accumulators, so the epilogue of tile i overlaps the
// MMAs of tile i + 1.
#pragma once
#include "ra_sm100.cuh"

namespace ra {
namespace ffn {

constexpr int BM = 128, BN = 256, BK = 64;
constexpr int NSTAGE = 4;
constexpr int NUM_THREADS = 256;
constexpr int WARP_TMA = 4, WARP_MMA = 5;
constexpr uint32_t TMEM_COLS = 512;

struct Layout {
  static constexpr int A_BYTES = BM * BK * 2;            // 16 KB, 128 rows x 128 B
  static constexpr int B_BYTES = BN * BK * 2;            // 32 KB, 256 rows x 128 B
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int BAR_OFF = NSTAGE * STAGE_BYTES;
  static constexpr int B_FULL = 0, B_EMPTY = NSTAGE, B_ACC_FULL = 2 * NSTAGE, B_ACC_EMPTY = B_ACC_FULL + 2,
                       B_DRAIN = B_ACC_EMPTY + 2, NUM_BARS = B_DRAIN + 1;
  static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;   // TMEM base, abort flag
  static constexpr int BYTES = MISC_OFF + 16;
  static constexpr int ALLOC = BYTES + 1024;                // room to align the base to 1024 B
};
static_assert(Layout::ALLOC <= 232448, "shared memory");

struct Params {
  int K;                 // reduction length (multiple of BK)
  int N;                 // output columns (multiple of 64)
  int rows;              // rows of the block per batch entry (c)
  int m_tiles_per_b;     // ceil(rows / BM)
  int m_tiles;           // B * m_tiles_per_b
  int n_tiles;           // ceil(N / BN)
  int n_items;           // m_tiles * n_tiles
  // A tile coordinates for (batch entry b, row tile tt, K offset k0):
  //   (k0 % a_kdim, a_row0 + tt * BM, b * a_outer_per_b + k0 / a_kdim)
  int a_kdim, a_row0, a_outer_per_b;
  // output row of (b, r): b * c_rows_per_b + c_row0 + r, row-major with ldc columns
  long long c_rows_per_b;
  long long c_row0;
  long long ldc;
  const float* bias;     // [N]
  __nv_bfloat16* c;
  int gelu;              // 1: exact GELU after the bias
};

__device__ __forceinline__ void item_coords(int w, const Params& p, int& b, int& tt, int& nt) {
  const int mt = w % p.m_tiles;
  nt = w / p.m_tiles;
  b = mt / p.m_tiles_per_b;
  tt = mt - b * p.m_tiles_per_b;
}

__device__ __forceinline__ float gelu_exact(float x) { return 0.5f * x * (1.f + erff(x * 0.70710678118654752f)); }

// ------------------------------------------------------------------ producer (1 thread)
__device__ void producer(const CUtensorMap* tm_a, const CUtensorMap* tm_b, const Params& p, uint32_t sbase,
                         volatile int* abort_flag) {
  using L = Layout;
  auto bar = [&](int i) { return sbase + L::BAR_OFF + 8u * i; };
  int stage = 0;
  uint32_t phase = 0, issued = 0, issued_parity = 0;
  bool ok = true;
  for (int w = blockIdx.x; w < p.n_items && ok; w += gridDim.x) {
    int b, tt, nt;
    item_coords(w, p, b, tt, nt);
    for (int k0 = 0; k0 < p.K; k0 += BK) {
      if (!mbar_wait(bar(L::B_EMPTY + stage), phase ^ 1u, abort_flag)) { ok = false; break; }
      const uint32_t st = sbase + stage * L::STAGE_BYTES;
      mbar_arrive_expect_tx(bar(L::B_FULL + stage), L::STAGE_BYTES);
      tma_load_3d(tm_a, st, bar(L::B_FULL + stage), k0 % p.a_kdim, p.a_row0 + tt * BM,
                  b * p.a_outer_per_b + k0 / p.a_kdim);
      tma_load_3d(tm_b, st + L::A_BYTES, bar(L::B_FULL + stage), k0, nt * BN, 0);
      issued |= 1u << stage;
      issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
      if (++stage == NSTAGE) {
        stage = 0;
        phase ^= 1u;
      }
    }
  }
  if (!ok) {   // let every copy this CTA started land before the CTA can exit
    for (int s = 0; s < NSTAGE; ++s)
      if (issued & (1u << s)) drain_wait(bar(L::B_FULL + s), (issued_parity >> s) & 1u);
  }
}

// ------------------------------------------------------------------ MMA issuer (1 thread)
__device__ void mma_issuer(const Params& p, uint32_t sbase, uint32_t tmem, volatile int* abort_flag) {
  using L = Layout;
  auto bar = [&](int i) { return sbase + L::BAR_OFF + 8u * i; };
  constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN, 0, 0);   // A, B both K-major
  int stage = 0;
  uint32_t phase = 0;
  uint32_t acc_phase[2] = {0, 0};
  int j = 0;
  for (int w = blockIdx.x; w < p.n_items; w += gridDim.x, ++j) {
    const int acc = j & 1;
    if (!mbar_wait(bar(L::B_ACC_EMPTY + acc), acc_phase[acc] ^ 1u, abort_flag)) break;
    acc_phase[acc] ^= 1u;
    tc_fence_after();
    const uint32_t d = tmem + acc * BN;
    bool ok = true;
    for (int k0 = 0; k0 < p.K; k0 += BK) {
      if (!mbar_wait(bar(L::B_FULL + stage), phase, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const uint32_t sa = sbase + stage * L::STAGE_BYTES, sb = sa + L::A_BYTES;
#pragma unroll
      for (int kk = 0; kk < BK / 16; ++kk)
        umma_ss(d, sdesc_sw128(sa + kk * 32, 16, 1024), sdesc_sw128(sb + kk * 32, 16, 1024), IDESC,
                (k0 > 0 || kk > 0) ? 1u : 0u);
      tc_commit(bar(L::B_EMPTY + stage));   // the stage is free once these MMAs have read it
      if (++stage == NSTAGE) {
        stage = 0;
        phase ^= 1u;
      }
    }
    if (!ok) break;
    tc_commit(bar(L::B_ACC_FULL + acc));
  }
  tc_commit(bar(L::B_DRAIN));   // every MMA issued so far has completed before TMEM is released
  drain_wait(bar(L::B_DRAIN), 0);
}

// ------------------------------------------------------------------ epilogue (128 threads)
__device__ void epilogue(const Params& p, uint32_t sbase, uint32_t tmem, volatile int* abort_flag) {
  using L = Layout;
  auto bar = [&](int i) { return sbase + L::BAR_OFF + 8u * i; };
  const int lane = threadIdx.x & 31;
  const int quarter = threadIdx.x >> 5;            // warps 0-3: TMEM lanes 32 * quarter + lane
  const int r = quarter * 32 + lane;               // row within the tile
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
  uint32_t acc_phase[2] = {0, 0};
  int j = 0;
  for (int w = blockIdx.x; w < p.n_items; w += gridDim.x, ++j) {
    const int acc = j & 1;
    if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_ACC_FULL + acc), acc_phase[acc], abort_flag))) return;
    acc_phase[acc] ^= 1u;
    tc_fence_after();
    int b, tt, nt;
    item_coords(w, p, b, tt, nt);
    const int row_in_block = tt * BM + r;
    const bool row_ok = row_in_block < p.rows;
    __nv_bfloat16* crow = p.c + (static_cast<long long>(b) * p.c_rows_per_b + p.c_row0 + row_in_block) * p.ldc;
    const int n_base = nt * BN;
#pragma unroll 1
    for (int ch = 0; ch < BN / 32; ++ch) {
      const int n0 = n_base + 32 * ch;
      if (n0 >= p.N) break;   // uniform: N is a multiple of 64
      uint32_t v[32];
      tmem_ld32(lane_base + acc * BN + 32 * ch, v);
      tmem_ld_wait();
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float2 bb = __ldg(reinterpret_cast<const float2*>(p.bias + n0) + i);
        float x0 = __uint_as_float(v[2 * i]) + bb.x, x1 = __uint_as_float(v[2 * i + 1]) + bb.y;
        if (p.gelu) {
          x0 = gelu_exact(x0);
          x1 = gelu_exact(x1);
        }
        pk[i] = pack_bf16x2(x0, x1);
      }
      if (row_ok) {
        uint4* dst = reinterpret_cast<uint4*>(crow + n0);
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(L::B_ACC_EMPTY + acc));   // 4 arrivals: the accumulator is free
  }
}

// ------------------------------------------------------------------ kernel
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b, const Params p) {
  using L = Layout;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int i = 0; i < L::NUM_BARS; ++i) {
      const bool acc_empty = i == L::B_ACC_EMPTY || i == L::B_ACC_EMPTY + 1;
      mbar_init(sbase + L::BAR_OFF + 8u * i, acc_empty ? 4 : 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == WARP_MMA) {
    tmem_alloc(smem_u32(tmem_holder), TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == WARP_TMA && (threadIdx.x & 31) == 0) {
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp < 4) {
    epilogue(p, sbase, tmem, abort_flag);
  } else if (warp == WARP_TMA) {
    if ((threadIdx.x & 31) == 0) producer(&tm_a, &tm_b, p, sbase, abort_flag);
    __syncwarp();
  } else if (warp == WARP_MMA) {
    if ((threadIdx.x & 31) == 0) mma_issuer(p, sbase, tmem, abort_flag);
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace ffn
}  // namespace ra
