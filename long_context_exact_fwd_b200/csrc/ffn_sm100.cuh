// Blockwise feedforward after attention, for sm_100a: one persistent TMA + tcgen05 launch that
// runs both matrix products of every ring block, with the bias / GELU epilogue fused.
//
// Page "精读笔记 · Ring Attention with Blockwise Transformers for Near-Infinite Context", §2.2
// (BPT): the feedforward of each attention sub-layer is computed block by block, so its largest
// activation is a block's hidden layer instead of the whole sequence's (2bsh instead of 8bsh
// bytes); §3.5 Algorithm 1: per layer each host's block goes through attention, then the
// feedforward.  Y = gelu(X W1^T + b1) W2^T + b2 with X the block's attention output, heads side
// by side per token; GELU in its exact form x Phi(x) (the pages name no activation).
//
// Work items (tiles of 256 rows x 256 columns):
//   GEMM 1 of block r: A = the attention output O [B][H][S][Dh] read in place (token rows of the
//           block; K index = head * Dh + d), B = W1 [f][h], epi = bias + GELU, C = Z_u [B][c][f];
//   GEMM 2 of block r: A = Z_u, B = W2 [h][f], epi = bias, C = the block's rows of Y [B][S][h];
// in the order GEMM 1 of block 0, then for r = 1, 2, ...: GEMM 1 of block r, GEMM 2 of block r - 1,
// and last GEMM 2 of the final block.  Z_u (u = block index in the launch mod nbuf, nbuf =
// min(3, D)) are block-sized hidden activations in the caller's workspace.  Dependencies, through
// per-row-tile counters in the workspace (cleared before the launch):
//   ready[u][m]    GEMM 1 tiles of row tile m that have stored their Z columns; a GEMM 2 tile of
//                  row tile m starts loading Z once all column tiles of its block are in;
//   consumed[u][m] GEMM 2 tiles of row tile m whose MMAs have read Z; a GEMM 1 tile nbuf blocks
//                  later overwrites those rows only once every one of them has.
// The lag puts a whole segment of other tiles between each tile and what it waits for: a block's
// GEMM 2 waits on GEMM 1 tiles taken a segment earlier, and with three buffers a GEMM 1 tile
// waits on GEMM 2 tiles two segments back.
// CTA pairs take items in that order from a per-launch counter as they become free (a fixed round
// robin let the pairs drift apart, since second-product tiles are four times longer, and left
// second-product tiles waiting on first-product tiles taken late: 4 % slower), and an item only
// waits on items before it, all taken by resident CTAs (one CTA per SM, grid <= SMs): every wait
// ends.  Every wait is bounded all the same (RA_ERR_TIMEOUT, then the CTA unwinds).
//
// A CTA pair (cluster of 2, tcgen05 cta_group::2) computes each 256-row x 256-column tile: each
// CTA loads its own 128 rows of A and its own 128 of the tile's 256 B rows (weight rows), and one
// M = 256, N = 256 MMA per 16-wide K step runs on both SMs, so an SM brings in 32 KiB per 64-wide K
// step for 512 tensor cycles (64 B per clock, against 96 for a single CTA with 128 x 256 tiles).
// Loads of both CTAs complete on the even CTA's barriers; the even CTA's one MMA thread issues
// every MMA and commits to barriers in both CTAs.  The even CTA's producer takes the tile numbers
// and hands each to every role of both CTAs through a ring of tile numbers in shared memory.
// CTA (384 threads): warps 0-7 epilogue (thread = output row = TMEM lane; warps w and w + 4 share
// lane quarter w, columns 0-127 and 128-255; the even CTA holds rows 0-127 of the tile, the odd one
// rows 128-255), warp 8 TMA producer (3-stage ring of 64 KiB: 128-wide K steps, so the MMA
// thread waits and commits once per 8 MMAs; 3 % faster than 64-wide steps in 6 stages; no
// multicast), warp 9 TMEM
// allocation (both CTAs) and, in the even CTA, the tcgen05.mma issue.
// TMEM per CTA: two 128 x 256 fp32 accumulators, so a tile's epilogue runs under the next tile's
// MMAs.
#pragma once
#include "ra_sm100.cuh"
#include "ra_work.cuh"

namespace ra {
namespace ffn {

constexpr int BM = 256, BN = 256, BK = 128;   // tile of a CTA pair, K step of a stage
constexpr int HALF = 128;                     // rows of A and of B per CTA
constexpr int NSTAGE = 3;
constexpr int EPI_WARPS = 8;        // two per TMEM lane quarter, each taking half of the columns
constexpr int NUM_THREADS = 384;
constexpr int WARP_TMA = 8, WARP_MMA = 9;   // warps 10-11 only complete the third warpgroup
constexpr int NITEM = 4;   // entries of the pair's ring of tile numbers
constexpr uint32_t TMEM_COLS = 512;

struct Layout {
  static constexpr int SUB_BYTES = HALF * 64 * 2;        // 128 rows x 64 columns (128 B, swizzled)
  static constexpr int A_BYTES = (BK / 64) * SUB_BYTES;  // 32 KB: this CTA's 128 rows of A
  static constexpr int B_BYTES = (BK / 64) * SUB_BYTES;  // 32 KB: this CTA's 128 of the 256 B rows
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int BAR_OFF = NSTAGE * STAGE_BYTES;
  // FULL: used in the even CTA (both CTAs' loads complete on it); EMPTY, ACC_FULL: in both CTAs
  // (the even CTA's MMA commits to both); ACC_EMPTY: in the even CTA (the epilogue warps of both
  // CTAs arrive)
  // ITEM_FULL: in both CTAs (the even CTA's producer publishes each tile number to both);
  // ITEM_EMPTY: in the even CTA (every reader of both CTAs arrives)
  static constexpr int B_FULL = 0, B_EMPTY = NSTAGE, B_ACC_FULL = 2 * NSTAGE, B_ACC_EMPTY = B_ACC_FULL + 2,
                       B_DRAIN = B_ACC_EMPTY + 2, B_ITEM_FULL = B_DRAIN + 1, B_ITEM_EMPTY = B_ITEM_FULL + NITEM,
                       NUM_BARS = B_ITEM_EMPTY + NITEM;
  // readers of a tile number: the even CTA's MMA thread and its epilogue warps, the odd CTA's
  // producer thread and its epilogue warps
  static constexpr uint32_t ITEM_READERS = 2 + 2 * EPI_WARPS;
  static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;   // TMEM base, abort flag, tile numbers
  static constexpr int ITEMS_OFF = MISC_OFF + 8;
  static constexpr int BYTES = ITEMS_OFF + 4 * NITEM;
  static constexpr int ALLOC = BYTES + 1024;                // room to align the base to 1024 B
};
static_assert(Layout::ALLOC <= 232448, "shared memory");

struct Params {
  int S, H, Dh, c, h, f;
  int r0, nblocks;       // ring blocks r0 .. r0 + nblocks - 1
  int mt_per_b;          // row tiles per batch entry: ceil(c / BM)  (BM = 256, a CTA pair)
  int MT;                // row tiles per block: B * mt_per_b
  int NT1, NT2;          // column tiles of GEMM 1 (f) and GEMM 2 (h)
  int per_block;         // MT * (NT1 + NT2)
  int n_items;           // nblocks * per_block
  int nbuf;              // hidden-activation buffers: min(3, D)
  int work_slot;         // this launch's work counter
  const float* b1;       // [f]
  const float* b2;       // [h]
  __nv_bfloat16* z;      // [nbuf][B][c][f] hidden activations
  __nv_bfloat16* y;      // [B][S][h]
  unsigned* ready;       // [nbuf][MT]
  unsigned* consumed;    // [nbuf][MT]
};

struct Tile {
  int blk, u;            // block index in the launch, its Z buffer
  int g;                 // 1: GEMM 1, 2: GEMM 2
  int mt, nt, b, tt;     // row tile in the block, column tile, batch entry, row tile in the entry
};

// Item w -> tile.  Segments: GEMM 1 of block 0; then (GEMM 1 of block k, GEMM 2 of block k - 1)
// for k = 1 .. nblocks - 1; then GEMM 2 of the last block.  Inside a segment the row tiles go
// fastest (consecutive CTA pairs share a weight slab in L2).  (Row tile by row tile, with each row
// tile's GEMM 2 tiles right behind its GEMM 1 tiles, measured 24 % slower: the pairs in flight then
// stream different weight slabs.)
__device__ __forceinline__ Tile decode(int w, const Params& p) {
  const int s1 = p.MT * p.NT1, s2 = p.MT * p.NT2;
  Tile t;
  int idx;
  if (w < s1) {
    t.blk = 0;
    t.g = 1;
    idx = w;
  } else {
    const int v = w - s1;
    const int q = v / (s1 + s2);
    const int off = v - q * (s1 + s2);
    if (q < p.nblocks - 1 && off < s1) {
      t.blk = q + 1;
      t.g = 1;
      idx = off;
    } else {
      t.blk = q;
      t.g = 2;
      idx = q < p.nblocks - 1 ? off - s1 : off;
    }
  }
  t.u = t.blk % p.nbuf;
  t.mt = idx % p.MT;
  t.nt = idx / p.MT;
  t.b = t.mt / p.mt_per_b;
  t.tt = t.mt - t.b * p.mt_per_b;
  return t;
}

__device__ __forceinline__ float gelu_exact(float x) { return 0.5f * x * (1.f + erff(x * 0.70710678118654752f)); }

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Bounded wait until *ctr >= target (acquire): RA_ERR_TIMEOUT and false after the time limit or
// once another warp of the CTA has given up.
__device__ __forceinline__ bool wait_count(const unsigned* ctr, unsigned target, volatile int* abort_flag) {
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 0;; ++it) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
    if (v >= target) return true;
    if ((it & 63u) == 63u) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > RA_WAIT_TIMEOUT_NS) break;
    }
    __nanosleep(64);
  }
  *abort_flag = 1;
  record_status(RA_ERR_TIMEOUT);
  return false;
}

__device__ __forceinline__ void signal_count(unsigned* ctr) {
  asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(ctr) : "memory");
}

// ------------------------------------------------------------------ CTA-pair primitives
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// The shared::cluster address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
  uint32_t d;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(saddr), "r"(rank));
  return d;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.aligned;\n\tbarrier.cluster.wait.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}
// 3-D tile load into this CTA's shared memory whose completion is counted on a barrier of the
// pair (the even CTA's): the cta_group::2 form, no multicast.
__device__ __forceinline__ void tma_load_3d_pair(const CUtensorMap* map, uint32_t dst, uint32_t bar_cluster, int c0,
                                                 int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void umma_ss_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on `bar_cluster` (a barrier of either CTA) once this thread's pair MMAs complete.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar_cluster) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar_cluster)
               : "memory");
}

// Tile numbers of the pair.  The even CTA's producer takes them from the launch's work counter
// (dynamic: a pair that finishes early takes the next tile, so the pairs do not drift apart the
// way a fixed round robin of tiles of unequal length makes them) and writes each into the same
// ring entry of both CTAs.  Readers wait on their own CTA's ITEM_FULL with cluster-scope acquire
// and arrive on the even CTA's ITEM_EMPTY.
__device__ __forceinline__ bool mbar_try_wait_acq_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_acq_cluster(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 0; it != 0xffffffffu; ++it) {
    if (mbar_try_wait_acq_cluster(bar, parity)) return true;
    if ((it & 127u) == 127u) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > RA_WAIT_TIMEOUT_NS) break;
    }
  }
  *abort_flag = 1;
  record_status(RA_ERR_TIMEOUT);
  return false;
}
__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

struct PairItems {
  uint32_t sbase;
  int k = 0;
  uint32_t ph = 0;
  __device__ __forceinline__ uint32_t bar(int i) const { return sbase + Layout::BAR_OFF + 8u * i; }
  __device__ __forceinline__ uint32_t slot() const { return sbase + Layout::ITEMS_OFF + 4u * k; }
  __device__ __forceinline__ void advance() {
    if (++k == NITEM) {
      k = 0;
      ph ^= 1u;
    }
  }
  // even CTA's producer: publish `item` to both CTAs once every reader has read the entry's last
  __device__ __forceinline__ bool push(int item, volatile int* abort_flag) {
    if (!mbar_wait(bar(Layout::B_ITEM_EMPTY + k), ph ^ 1u, abort_flag)) return false;
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(slot()), "r"(static_cast<uint32_t>(item)) : "memory");
    st_cluster_u32(map_to_rank(slot(), 1), static_cast<uint32_t>(item));
    mbar_arrive(bar(Layout::B_ITEM_FULL + k));
    mbar_arrive_cluster(map_to_rank(bar(Layout::B_ITEM_FULL + k), 1));   // release: the store above first
    advance();
    return true;
  }
  // one reading thread (arrives once)
  __device__ __forceinline__ bool pop(int& item, volatile int* abort_flag) {
    if (!mbar_wait_acq_cluster(bar(Layout::B_ITEM_FULL + k), ph, abort_flag)) return false;
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(slot()) : "memory");
    item = static_cast<int>(v);
    mbar_arrive_cluster(map_to_rank(bar(Layout::B_ITEM_EMPTY + k), 0));
    advance();
    return true;
  }
  // a whole warp reads, lane 0 arrives once; uniform outcome
  __device__ __forceinline__ bool pop_warp(int& item, volatile int* abort_flag) {
    if (!__all_sync(0xffffffffu, mbar_wait_acq_cluster(bar(Layout::B_ITEM_FULL + k), ph, abort_flag))) return false;
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(slot()) : "memory");
    item = static_cast<int>(v);
    __syncwarp();
    if ((threadIdx.x & 31u) == 0u) mbar_arrive_cluster(map_to_rank(bar(Layout::B_ITEM_EMPTY + k), 0));
    advance();
    return true;
  }
};

// ------------------------------------------------------------------ producer (1 thread per CTA)
__device__ void producer(const CUtensorMap* tm_x, const CUtensorMap* tm_w1, const CUtensorMap* tm_z,
                         const CUtensorMap* tm_w2, const Params& p, uint32_t sbase, uint32_t rank,
                         volatile int* abort_flag) {
  using L = Layout;
  auto bar = [&](int i) { return sbase + L::BAR_OFF + 8u * i; };
  int stage = 0;
  uint32_t phase = 0, issued = 0, issued_parity = 0;
  bool ok = true;
  PairItems items{sbase};
  int w = rank == 0 ? work_fetch(p.work_slot) : 0;
  for (;;) {
    if (rank == 0 ? !items.push(w, abort_flag) : !items.pop(w, abort_flag)) {
      ok = false;
      break;
    }
    if (w >= p.n_items) break;
    const int w_next = rank == 0 ? work_fetch(p.work_slot) : 0;   // in flight while this tile's loads issue
    const Tile t = decode(w, p);
    const int r = p.r0 + t.blk;
    const int K = t.g == 1 ? p.h : p.f;
    const int row = t.tt * BM + rank * HALF;   // this CTA's rows of the tile, within the batch entry
    if (t.g == 2) {   // every column tile of this row tile's hidden activation is stored (both CTAs)
      if (!wait_count(p.ready + t.u * p.MT + t.mt, static_cast<unsigned>(2 * p.NT1 * (t.blk / p.nbuf + 1)), abort_flag)) {
        ok = false;
        break;
      }
      fence_proxy_async_global();   // the generic-proxy stores of Z before these TMA reads
    }
    for (int k0 = 0; k0 < K; k0 += BK) {
      if (!mbar_wait(bar(L::B_EMPTY + stage), phase ^ 1u, abort_flag)) { ok = false; break; }
      const uint32_t st = sbase + stage * L::STAGE_BYTES;
      const uint32_t full = map_to_rank(bar(L::B_FULL + stage), 0);   // the even CTA's barrier
      // 64-column sub-steps (the last step of a K that is an odd multiple of 64 has one: a load
      // past the end of the attention output's heads would read the next batch entry's)
      const int nsub = K - k0 >= BK ? BK / 64 : 1;
      if (rank == 0) mbar_arrive_expect_tx(bar(L::B_FULL + stage), 4 * nsub * L::SUB_BYTES);   // both CTAs' bytes
      for (int j = 0; j < nsub; ++j) {
        const int kj = k0 + 64 * j;
        const uint32_t sj = st + j * L::SUB_BYTES;
        if (t.g == 1) {
          tma_load_3d_pair(tm_x, sj, full, kj % p.Dh, r * p.c + row, t.b * p.H + kj / p.Dh);
          tma_load_3d_pair(tm_w1, sj + L::A_BYTES, full, kj, t.nt * BN + rank * HALF, 0);
        } else {
          tma_load_3d_pair(tm_z, sj, full, kj, row, t.u * (p.MT / p.mt_per_b) + t.b);
          tma_load_3d_pair(tm_w2, sj + L::A_BYTES, full, kj, t.nt * BN + rank * HALF, 0);
        }
      }
      issued |= 1u << stage;
      issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
      if (++stage == NSTAGE) {
        stage = 0;
        phase ^= 1u;
      }
    }
    if (!ok) break;
    w = w_next;
  }
  work_done(p.work_slot);   // each CTA once (the odd one after reading the end marker)
  if (!ok && rank == 0) {   // let every copy the pair started land (they count on these barriers)
    for (int s = 0; s < NSTAGE; ++s)
      if (issued & (1u << s)) drain_wait(bar(L::B_FULL + s), (issued_parity >> s) & 1u);
  }
}

// ------------------------------------------------------------------ MMA issuer (1 thread, even CTA)
__device__ void mma_issuer(const Params& p, uint32_t sbase, uint32_t tmem, volatile int* abort_flag) {
  using L = Layout;
  auto bar = [&](int i) { return sbase + L::BAR_OFF + 8u * i; };
  auto both = [&](int i) {   // commit to barrier i of each CTA
    tc_commit_pair(map_to_rank(bar(i), 0));
    tc_commit_pair(map_to_rank(bar(i), 1));
  };
  constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN, 0, 0);   // M = 256 over the pair, A, B K-major
  int stage = 0;
  uint32_t phase = 0;
  uint32_t acc_phases = 0;   // bit a: phase of accumulator a
  PairItems items{sbase};
  for (int j = 0;; ++j) {
    int w;
    if (!items.pop(w, abort_flag) || w >= p.n_items) break;
    const Tile t = decode(w, p);
    const int K = t.g == 1 ? p.h : p.f;
    const int acc = j & 1;
    if (!mbar_wait(bar(L::B_ACC_EMPTY + acc), ((acc_phases >> acc) & 1u) ^ 1u, abort_flag)) break;
    acc_phases ^= 1u << acc;
    tc_fence_after();
    const uint32_t d = tmem + acc * BN;
    bool ok = true;
    for (int k0 = 0; k0 < K; k0 += BK) {
      if (!mbar_wait(bar(L::B_FULL + stage), phase, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const uint32_t sa = sbase + stage * L::STAGE_BYTES, sb = sa + L::A_BYTES;
      const int nk = K - k0 >= BK ? BK / 16 : 4;   // 16-wide MMAs of this step (4 on a 64-wide tail)
#pragma unroll
      for (int kk = 0; kk < BK / 16; ++kk) {
        const uint32_t off = (kk >> 2) * L::SUB_BYTES + (kk & 3) * 32;
        if (kk < nk)
          umma_ss_pair(d, sdesc_sw128(sa + off, 16, 1024), sdesc_sw128(sb + off, 16, 1024), IDESC,
                       (k0 > 0 || kk > 0) ? 1u : 0u);
      }
      both(L::B_EMPTY + stage);   // the stage is free in both CTAs once these MMAs have read it
      if (++stage == NSTAGE) {
        stage = 0;
        phase ^= 1u;
      }
    }
    if (!ok) break;
    both(L::B_ACC_FULL + acc);
  }
  tc_commit_pair(map_to_rank(bar(L::B_DRAIN), 0));   // every MMA issued so far has completed
  drain_wait(bar(L::B_DRAIN), 0);
}

// ------------------------------------------------------------------ epilogue (256 threads per CTA)
__device__ void epilogue(const Params& p, uint32_t sbase, uint32_t tmem, uint32_t rank, volatile int* abort_flag) {
  using L = Layout;
  auto bar = [&](int i) { return sbase + L::BAR_OFF + 8u * i; };
  constexpr uint32_t NT = EPI_WARPS * 32;          // epilogue threads (named barrier 1)
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int quarter = warp & 3;                    // TMEM lanes 32 * quarter + lane
  const int col0 = (warp >> 2) * (BN / 2);         // this warp's half of the tile's columns
  const int r = static_cast<int>(rank) * HALF + quarter * 32 + lane;   // row within the pair's tile
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
  uint32_t acc_phases = 0;   // bit a: phase of accumulator a
  PairItems items{sbase};
  for (int j = 0;; ++j) {
    int w;
    // uniform outcome across the epilogue warps (the named barriers below need all of them)
    const bool got = items.pop_warp(w, abort_flag);
    if (!named_bar_and(1, NT, got && w < p.n_items)) return;
    const Tile t = decode(w, p);
    const int acc = j & 1;
    // uniform outcomes across the four warps: the named barriers below need all of them
    if (!named_bar_and(1, NT, mbar_wait(bar(L::B_ACC_FULL + acc), (acc_phases >> acc) & 1u, abort_flag))) return;
    acc_phases ^= 1u << acc;
    tc_fence_after();
    const int row_in_block = t.tt * BM + r;
    const bool row_ok = row_in_block < p.c;
    __nv_bfloat16* crow;
    const float* bias;
    int N;
    if (t.g == 1) {
      // Z_u rows of this row tile are overwritten only once the GEMM 2 tiles of the block nbuf
      // before have read them
      bool go = true;
      if (t.blk >= p.nbuf && threadIdx.x == 0)
        go = wait_count(p.consumed + t.u * p.MT + t.mt, static_cast<unsigned>(2 * p.NT2 * (t.blk / p.nbuf)), abort_flag);
      if (!named_bar_and(1, NT, go)) return;
      crow = p.z + ((static_cast<long long>(t.u) * (p.MT / p.mt_per_b) + t.b) * p.c + row_in_block) * p.f;
      bias = p.b1;
      N = p.f;
    } else {
      // this tile's MMAs have read its Z rows in this CTA: they may be overwritten
      if (threadIdx.x == 0) signal_count(p.consumed + t.u * p.MT + t.mt);
      crow = p.y + (static_cast<long long>(t.b) * p.S + static_cast<long long>(p.r0 + t.blk) * p.c + row_in_block) * p.h;
      bias = p.b2;
      N = p.h;
    }
    const int n_base = t.nt * BN + col0;
#pragma unroll 1
    for (int ch = 0; ch < BN / 64; ++ch) {
      const int n0 = n_base + 32 * ch;
      if (n0 >= N) break;   // uniform: N is a multiple of 64
      uint32_t v[32];
      tmem_ld32(lane_base + acc * BN + col0 + 32 * ch, v);
      tmem_ld_wait();
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float2 bb = __ldg(reinterpret_cast<const float2*>(bias + n0) + i);
        float x0 = __uint_as_float(v[2 * i]) + bb.x, x1 = __uint_as_float(v[2 * i + 1]) + bb.y;
        if (t.g == 1) {
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
    // 2 * EPI_WARPS arrivals on the even CTA's barrier: the accumulator is free
    if (lane == 0) mbar_arrive_cluster(map_to_rank(bar(L::B_ACC_EMPTY + acc), 0));
    if (t.g == 1) {   // publish this CTA's half of the tile's Z columns
      fence_proxy_async_global();   // for the TMA (async proxy) reads that follow elsewhere
      __threadfence();
      named_bar_sync(1, NT);
      if (threadIdx.x == 0) signal_count(p.ready + t.u * p.MT + t.mt);
    }
  }
}

// ------------------------------------------------------------------ kernel (clusters of 2 CTAs)
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    ffn_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w1,
               const __grid_constant__ CUtensorMap tm_z, const __grid_constant__ CUtensorMap tm_w2, const Params p) {
  using L = Layout;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);
  const int warp = threadIdx.x >> 5;
  const uint32_t rank = cluster_rank();
  if (threadIdx.x == 0) {
    for (int i = 0; i < L::NUM_BARS; ++i) {
      const bool acc_empty = i == L::B_ACC_EMPTY || i == L::B_ACC_EMPTY + 1;
      const bool item_empty = i >= L::B_ITEM_EMPTY && i < L::B_ITEM_EMPTY + NITEM;
      mbar_init(sbase + L::BAR_OFF + 8u * i, acc_empty ? 2 * EPI_WARPS : (item_empty ? L::ITEM_READERS : 1));
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == WARP_MMA) {   // both CTAs, the same warp: the pair's TMEM
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_holder)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  if (warp == WARP_TMA && (threadIdx.x & 31) == 0) {
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w1);
    tma_prefetch_desc(&tm_z);
    tma_prefetch_desc(&tm_w2);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();   // both CTAs' barriers are initialised before either CTA touches the other's
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp < EPI_WARPS) {
    epilogue(p, sbase, tmem, rank, abort_flag);
  } else if (warp == WARP_TMA) {
    if ((threadIdx.x & 31) == 0) producer(&tm_x, &tm_w1, &tm_z, &tm_w2, p, sbase, rank, abort_flag);
    __syncwarp();
  } else if (warp == WARP_MMA) {
    if (rank == 0 && (threadIdx.x & 31) == 0) mma_issuer(p, sbase, tmem, abort_flag);
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();   // the pair's MMAs have drained and both epilogues are done with TMEM
  if (warp == WARP_MMA) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
  }
  cluster_sync();   // neither CTA leaves while the other may still address its shared memory
}

}  // namespace ffn
}  // namespace ra
